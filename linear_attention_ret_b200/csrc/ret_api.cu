// C ABI of libret.so (declared in include/ret.h): host-side validation, kernel
// selection and launch. One translation unit holds every kernel so that they
// share the module-scope device error word.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "simt.cuh"
#include "decode.cuh"
#include "tc_chunk.cuh"
#include "seqpar.cuh"
#include "backward.cuh"
#include "norm.cuh"

using namespace ret;

namespace {

constexpr int kMaxGridY = 65535;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline ret_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? RET_OK : RET_ERR_CUDA;
}

ret_status check_common(int B, int H, int N, int dk, int dv, int dt) {
    if (dt != RET_F32 && dt != RET_BF16) return RET_ERR_DTYPE;
    if (B <= 0 || H <= 0 || N < 0 || dk <= 0 || dv <= 0) return RET_ERR_SHAPE;
    if ((long long)B * H > kMaxGridY) return RET_ERR_UNSUPPORTED;
    return RET_OK;
}

// state_out <- state_in (or zeros) for an empty sequence.
ret_status empty_sequence_state(const float* state_in, float* state_out, int B, int H, int dk, int dv,
                                cudaStream_t st) {
    if (state_out == nullptr) return RET_OK;
    const size_t bytes = sizeof(float) * (size_t)B * H * dk * dv;
    cudaError_t e = state_in ? (state_in == state_out ? cudaSuccess
                                                      : cudaMemcpyAsync(state_out, state_in, bytes,
                                                                        cudaMemcpyDeviceToDevice, st))
                             : cudaMemsetAsync(state_out, 0, bytes, st);
    return e == cudaSuccess ? RET_OK : RET_ERR_CUDA;
}

template <typename T, bool GATED>
ret_status launch_chunkwise_simt(const void* q, const void* k, const void* v, const float* decay,
                                 void* o, const float* state_in, float* state_out,
                                 int B, int H, int N, int dk, int dv, int chunk, cudaStream_t st) {
    auto kern = chunkwise_simt_kernel<T, GATED>;
    const size_t smem = chunkwise_simt_smem_bytes(dk);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return RET_ERR_CUDA;
    dim3 grid((dv + kCwV - 1) / kCwV, B * H);
    kern<<<grid, kCwThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                         static_cast<const T*>(v), decay, state_in, state_out,
                                         static_cast<T*>(o), H, N, dk, dv, chunk);
    return launch_status();
}

template <bool GATED>
ret_status chunkwise_entry(const void* q, const void* k, const void* v, const float* decay,
                           void* o, const float* state_in, float* state_out,
                           int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (chunk <= 0) return RET_ERR_SHAPE;
    if (dk > 256) return RET_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (N == 0) return empty_sequence_state(state_in, state_out, B, H, dk, dv, st);
    if (!q || !k || !v || !decay || !o) return RET_ERR_NULL;
    if (tc_chunk_supported(dk, dv, chunk, dt == RET_BF16)) {
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RET_ERR_ALIGN;
        return tc_chunk_launch<GATED>(q, k, v, decay, o, state_in, state_out, B, H, N, dk, dv, st);
    }
    if (dt == RET_F32)
        return launch_chunkwise_simt<float, GATED>(q, k, v, decay, o, state_in, state_out, B, H, N, dk, dv,
                                                   chunk, st);
    return launch_chunkwise_simt<__nv_bfloat16, GATED>(q, k, v, decay, o, state_in, state_out, B, H, N, dk,
                                                       dv, chunk, st);
}

// End state of a sequence from a zero start and log2 of its total decay, without outputs.
template <bool GATED>
ret_status chunkwise_state_entry(const void* k, const void* v, const float* decay, float* state_out, float* log2_decay,
                                 int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (chunk <= 0) return RET_ERR_SHAPE;
    if (dk > 256) return RET_ERR_UNSUPPORTED;
    if (!state_out || !log2_decay) return RET_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    if (N == 0) {
        if (cudaMemsetAsync(log2_decay, 0, sizeof(float) * (size_t)B * H, st) != cudaSuccess) return RET_ERR_CUDA;
        return empty_sequence_state(nullptr, state_out, B, H, dk, dv, st);
    }
    if (!k || !v || !decay) return RET_ERR_NULL;
    const bool tc = tc_chunk_supported(dk, dv, chunk, dt == RET_BF16);
    if (tc && (!aligned16(k) || !aligned16(v))) return RET_ERR_ALIGN;
    segment_log2_decay_kernel<GATED><<<B * H, 256, 0, st>>>(decay, log2_decay, H, N);
    if (cudaGetLastError() != cudaSuccess) return RET_ERR_CUDA;
    if (tc) return tc_state_launch<GATED>(k, v, decay, state_out, B, H, N, dk, dv, st);
    // CUDA-core path: the chunkwise kernel with its outputs sent to scratch (K stands in for Q)
    void* o = nullptr;
    if (cudaMallocAsync(&o, (size_t)B * H * N * dv * (dt == RET_F32 ? 4 : 2), st) != cudaSuccess) return RET_ERR_CUDA;
    const ret_status r =
        dt == RET_F32
            ? launch_chunkwise_simt<float, GATED>(k, k, v, decay, o, nullptr, state_out, B, H, N, dk, dv, chunk, st)
            : launch_chunkwise_simt<__nv_bfloat16, GATED>(k, k, v, decay, o, nullptr, state_out, B, H, N, dk, dv,
                                                          chunk, st);
    if (cudaFreeAsync(o, st) != cudaSuccess) return RET_ERR_CUDA;
    return r;
}

// ------------------------------------------------------------------ backward (see backward.cuh)

inline int grid_for(size_t n) { return (int)std::min<size_t>((n + kBwdThreads - 1) / kBwdThreads, 8 * tc::sm_count()); }
// Row kernels: one warp per `per_warp` rows, up to 32 blocks per SM.
inline unsigned rows_grid(size_t rows, int per_warp = 1) {
    const size_t warps = (rows + per_warp - 1) / per_warp;
    return (unsigned)std::min<size_t>((warps + kBwdWarps - 1) / kBwdWarps, (size_t)32 * tc::sm_count());
}
inline bool whole_chunks(size_t elems, size_t elt) { return (elems * elt) % 16 == 0; }

template <typename T>
ret_status sum_flip(const T* parts, int P, size_t part_elems, T* out, int BH, int N, int d, bool flip, cudaStream_t st) {
    const size_t rows = (size_t)BH * N;
    if (whole_chunks(d, sizeof(T)) && whole_chunks(part_elems, sizeof(T)) && aligned16(parts) && aligned16(out))
        sum_flip_kernel<T, true><<<rows_grid(rows), kBwdThreads, 0, st>>>(parts, P, part_elems, out, N, d, flip, rows);
    else
        sum_flip_kernel<T, false><<<rows_grid(rows), kBwdThreads, 0, st>>>(parts, P, part_elems, out, N, d, flip, rows);
    return launch_status();
}

template <typename T>
ret_status slice_flip(const void* src, void* dst, int BH, int N, int d_src, int c0, int w, bool flip, cudaStream_t st) {
    const size_t rows = (size_t)BH * N;
    const T* s = static_cast<const T*>(src);
    T* d = static_cast<T*>(dst);
    if (whole_chunks(d_src, sizeof(T)) && whole_chunks(c0, sizeof(T)) && whole_chunks(w, sizeof(T)) && aligned16(s) &&
        aligned16(d))
        slice_flip_kernel<T, true><<<rows_grid(rows, kCopyRows), kBwdThreads, 0, st>>>(s, d, N, d_src, c0, w, flip,
                                                                                       rows);
    else
        slice_flip_kernel<T, false><<<rows_grid(rows, kCopyRows), kBwdThreads, 0, st>>>(s, d, N, d_src, c0, w, flip,
                                                                                        rows);
    return launch_status();
}

template <typename T, bool GATED>
ret_status decay_grad(const T* q, const T* dq, const T* k, const T* dk, const float* decay, float* out, int BH, int H,
                      int N, int dk_dim, cudaStream_t st) {
    if (!GATED && cudaMemsetAsync(out, 0, sizeof(float) * (size_t)H, st) != cudaSuccess) return RET_ERR_CUDA;
    const int ntiles = (N + kGradTokens - 1) / kGradTokens;
    const dim3 grid((unsigned)ntiles, (unsigned)BH);
    const bool vec = whole_chunks(dk_dim, sizeof(T)) && aligned16(q) && aligned16(dq) && aligned16(k) && aligned16(dk);
    const int C = vec ? dk_dim / RowIo<T, true>::kE : 0;  // 16-byte chunks per row
    int lc = 0;
    while ((1 << lc) < C) ++lc;
    if (vec && C == (1 << lc) && C <= 32) {
        // all of a tile's loads in flight; gated: in-tile suffix sums and tile totals, then
        // the later tiles' totals added by a second, fully parallel kernel
        float* tot = nullptr;
        if (GATED && cudaMallocAsync(reinterpret_cast<void**>(&tot), sizeof(float) * (size_t)BH * ntiles, st) !=
                         cudaSuccess)
            return RET_ERR_CUDA;
        decay_grad_flat_kernel<T, GATED><<<grid, kBwdThreads, 0, st>>>(q, dq, k, dk, decay, out, tot, H, N, lc);
        ret_status r = launch_status();
        if (GATED) {
            if (r == RET_OK) {
                const dim3 g2((unsigned)((ntiles + kCarryTiles - 1) / kCarryTiles), (unsigned)BH);
                gate_grad_carry_kernel<<<g2, kBwdThreads, 0, st>>>(out, tot, N, ntiles);
                r = launch_status();
            }
            if (cudaFreeAsync(tot, st) != cudaSuccess && r == RET_OK) r = RET_ERR_CUDA;
        }
        return r;
    }
    if (vec)
        decay_grad_kernel<T, true, GATED><<<grid, kBwdThreads, 0, st>>>(q, dq, k, dk, decay, out, H, N, dk_dim);
    else
        decay_grad_kernel<T, false, GATED><<<grid, kBwdThreads, 0, st>>>(q, dq, k, dk, decay, out, H, N, dk_dim);
    ret_status r = launch_status();
    if (GATED && r == RET_OK) {
        gate_grad_scan_kernel<<<(unsigned)BH, kScanThreads, 0, st>>>(out, N);
        r = launch_status();
    }
    return r;
}

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Library streams per device, with events, for the steps of the backward that run side by
// side: kAuxHi streams of the device's greatest priority for the passes that the decay
// gradient waits for, and one of the least priority for the pass that it does not wait for.
// Held under the mutex from the first fork to the last join, so calls from several host
// threads do not interleave their events.
constexpr int kAuxHi = 4, kAuxStreams = kAuxHi + 1, kAuxEvents = kAuxStreams + 1;
struct AuxStreams {
    cudaStream_t s[kAuxStreams] = {};
    cudaEvent_t ev[kAuxEvents] = {};
};
constexpr int kMaxDevices = 64;
inline std::mutex& aux_mutex() {
    static std::mutex m;
    return m;
}
inline void destroy_aux(AuxStreams& n) {
    for (cudaEvent_t e : n.ev)
        if (e) cudaEventDestroy(e);
    for (cudaStream_t x : n.s)
        if (x) cudaStreamDestroy(x);
}
inline AuxStreams* aux_streams() {
    static AuxStreams aux[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    AuxStreams& a = aux[dev];
    if (!a.s[0]) {  // publish only once every stream and event exists
        AuxStreams n;
        bool ok = true;
        int least = 0, greatest = 0;
        ok = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess;
        for (int i = 0; i < kAuxStreams; ++i)
            ok = ok && cudaStreamCreateWithPriority(&n.s[i], cudaStreamNonBlocking, i < kAuxHi ? greatest : least) ==
                           cudaSuccess;
        for (cudaEvent_t& e : n.ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            destroy_aux(n);
            return nullptr;
        }
        a = n;
    }
    return &a;
}

// The backward on the tensor-core path: every launch (the dQ pieces, the dK pieces and dV,
// each with q/k widths of at most 256 read in place through row-strided tensor maps) is a
// tensor-core launch. dK and dV run on the time-reversed kernels, so nothing is copied.
inline bool backward_on_tensor_cores(int dk, int dv, int chunk, ret_dtype dt) {
    if (dt != RET_BF16 || !tc_chunk_supported(dk, dv, chunk, true)) return false;  // dV: widths dk, values dv
    for (int c0 = 0; c0 < dv; c0 += 256)
        if (!tc_chunk_supported(std::min(256, dv - c0), dk, chunk, true)) return false;  // dQ, dK pieces
    return true;
}

// Kernel launches of one backward call on the tensor-core path.
inline int backward_tc_launches(int B, int H, int N, int dk, int dv, bool gated, bool ddecay) {
    const int P = (dv + 255) / 256, conc = 2 * P + 1;
    int n = 0;
    for (int p = 0; p < P; ++p) n += 2 * tc_chunk_launches(B, H, N, std::min(256, dv - 256 * p), dk, conc);
    n += tc_chunk_launches(B, H, N, dk, dv, conc);  // dV
    n += ddecay ? (gated ? 2 : 1) : 0;              // decay gradient (gated: and its suffix sum)
    return n;
}

// The backward on the tensor-core path as a small graph of steps. Library streams h0..h3 (the
// greatest priority) take the passes that the decay gradient needs, the low-priority stream
// lo takes dV, which nothing in the call waits for:
//   st: zero dq, dk | fork | wait h0..h3 -> dgamma/dg | wait lo
//   h0, h1: dQ pieces 0, 1 (adding onto dq; more pieces alternate between the two)
//   h2, h3: dK pieces 0, 1 (reversed, adding onto dk)
//   lo:     dV (reversed)
// All passes start together and the block scheduler serves the high-priority passes first, so
// dV fills the SMs that they leave free and the decay gradient runs beside the end of dV. With
// one piece the dQ and dK calls store dq and dk directly, with no zeroing. dQ = forward(dO, V,
// K); dK = reversed forward(V, dO, Q); dV = reversed forward(K, Q, dO), each with the caller's
// gamma or gates as they are.
template <typename T, bool GATED>
ret_status backward_tc(const void* q, const void* k, const void* v, const float* decay, const void* dout,
                       void* dq, void* dk_out, void* dv_out, float* ddecay, int B, int H, int N, int dk, int dv,
                       cudaStream_t st) {
    const size_t nQ = (size_t)B * H * N * dk;
    const int pw = 256, P = (dv + pw - 1) / pw, conc = 2 * P + 1;
    ret_status r = RET_OK;
    auto ok = [&](ret_status x) { if (r == RET_OK) r = x; return r == RET_OK; };
    auto cu = [&](cudaError_t e) { return ok(e == cudaSuccess ? RET_OK : RET_ERR_CUDA); };
    std::lock_guard<std::mutex> lock(aux_mutex());
    AuxStreams* a = aux_streams();
    if (!a) return RET_ERR_CUDA;
    cudaStream_t* hi = a->s;
    cudaStream_t lo = a->s[kAuxHi];
    cudaEvent_t ev_fork = a->ev[0];
    cudaEvent_t* ev_done = a->ev + 1;  // one per library stream, after its last step
    // With several pieces, dq and dk start at zero and every piece adds its output tiles onto
    // them (in L2, in bf16, rounded once per addition): with two pieces each element is
    // round(a + b), whatever order the pieces' additions take.
    if (P > 1) {
        cu(cudaMemsetAsync(dq, 0, nQ * sizeof(T), st));
        cu(cudaMemsetAsync(dk_out, 0, nQ * sizeof(T), st));
    }
    // one piece of a dv contraction: queries x[:, c0:c0+w], keys y[:, c0:c0+w] (rows dv apart), values z
    auto piece = [&](bool rev, const void* x, const void* y, const void* z, void* out, int p, cudaStream_t s) {
        const int c0 = p * pw, w = std::min(pw, dv - c0);
        const void* xp = static_cast<const T*>(x) + c0;
        const void* yp = static_cast<const T*>(y) + c0;
        return ok(rev ? tc_chunk_launch<GATED, true>(xp, yp, z, decay, out, nullptr, nullptr, B, H, N, w, dk, s, dv,
                                                     dv, conc, P > 1)
                      : tc_chunk_launch<GATED, false>(xp, yp, z, decay, out, nullptr, nullptr, B, H, N, w, dk, s, dv,
                                                      dv, conc, P > 1));
    };
    if (r == RET_OK && cu(cudaEventRecord(ev_fork, st)))
        for (int i = 0; i < kAuxStreams && r == RET_OK; ++i) cu(cudaStreamWaitEvent(a->s[i], ev_fork, 0));
    // issue order: dQ pieces, dK pieces, then dV
    for (int p = 0; p < P && r == RET_OK; ++p) piece(false, dout, v, k, dq, p, hi[p % 2]);
    for (int p = 0; p < P && r == RET_OK; ++p) piece(true, v, dout, q, dk_out, p, hi[2 + p % 2]);
    if (r == RET_OK)
        ok(tc_chunk_launch<GATED, true>(k, q, dout, decay, dv_out, nullptr, nullptr, B, H, N, dk, dv, lo, 0, 0, conc));
    // join every library stream back into st whatever happened: the high-priority ones before
    // the decay gradient (it reads dq and dk), lo after it
    bool joined = true;
    for (int i = 0; i < kAuxStreams; ++i) joined = joined && cudaEventRecord(ev_done[i], a->s[i]) == cudaSuccess;
    for (int i = 0; i < kAuxHi; ++i) joined = joined && cudaStreamWaitEvent(st, ev_done[i], 0) == cudaSuccess;
    if (r == RET_OK && joined && ddecay)
        ok(decay_grad<T, GATED>(static_cast<const T*>(q), static_cast<const T*>(dq), static_cast<const T*>(k),
                                static_cast<const T*>(dk_out), decay, ddecay, B * H, H, N, dk, st));
    joined = joined && cudaStreamWaitEvent(st, ev_done[kAuxHi], 0) == cudaSuccess;
    if (!joined) {
        // the library streams could not be ordered before st: wait for them
        for (int i = 0; i < kAuxStreams; ++i) cudaStreamSynchronize(a->s[i]);
        ok(RET_ERR_CUDA);
    }
    return r;
}

template <typename T, bool GATED>
ret_status backward_impl(const void* q, const void* k, const void* v, const float* decay, const void* dout, void* dq,
                         void* dk_out, void* dv_out, float* ddecay, int B, int H, int N, int dk, int dv, int chunk,
                         ret_dtype dt, cudaStream_t st) {
    const int BH = B * H;
    const size_t nQ = (size_t)BH * N * dk, nV = (size_t)BH * N * dv;
    const int pw = dv <= 256 ? dv : 256;  // width of one piece of the dv contraction
    const int P = (dv + pw - 1) / pw;
    if (backward_on_tensor_cores(dk, dv, chunk, dt))
        return backward_tc<T, GATED>(q, k, v, decay, dout, dq, dk_out, dv_out, ddecay, B, H, N, dk, dv, st);
    // scratch: reversed Q, K, V, dO; two piece buffers; per-piece outputs; reversed dV; reversed gates
    size_t off[9], bytes = 0;
    const size_t sz[9] = {nQ * sizeof(T), nQ * sizeof(T), nV * sizeof(T), nV * sizeof(T),
                          P > 1 ? (size_t)BH * N * pw * sizeof(T) : 0, P > 1 ? (size_t)BH * N * pw * sizeof(T) : 0,
                          (size_t)P * nQ * sizeof(T),
                          nV * sizeof(T), GATED ? (size_t)BH * N * sizeof(float) : 0};
    for (int i = 0; i < 9; ++i) {
        off[i] = bytes;
        bytes += align256(sz[i]);
    }
    tc::keep_pool_memory();
    uint8_t* sc = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void**>(&sc), bytes, st) != cudaSuccess) return RET_ERR_CUDA;
    T* Qf = reinterpret_cast<T*>(sc + off[0]);
    T* Kf = reinterpret_cast<T*>(sc + off[1]);
    T* Vf = reinterpret_cast<T*>(sc + off[2]);
    T* dOf = reinterpret_cast<T*>(sc + off[3]);
    T* pa = reinterpret_cast<T*>(sc + off[4]);
    T* pb = reinterpret_cast<T*>(sc + off[5]);
    T* parts = reinterpret_cast<T*>(sc + off[6]);
    T* Rf = reinterpret_cast<T*>(sc + off[7]);
    float* gf = reinterpret_cast<float*>(sc + off[8]);
    ret_status r = RET_OK;
    auto ok = [&](ret_status x) { if (r == RET_OK) r = x; return r == RET_OK; };
    auto fwd = [&](const void* fq, const void* fk, const void* fv, const float* dec, void* fo, int wq, int wv) {
        return ok(chunkwise_entry<GATED>(fq, fk, fv, dec, fo, nullptr, nullptr, B, H, N, wq, wv, chunk, dt, st));
    };
    // All pieces of a dv contraction, copied out first: forward(a[:, c0:c0+w], b[:, c0:c0+w], c)
    // into parts[p], a and b dv wide.
    auto pieces = [&](const void* a, const void* b, const void* c, const float* dec) {
        for (int p = 0; p < P && r == RET_OK; ++p) {
            const int c0 = p * pw, w = std::min(pw, dv - c0);
            ok(slice_flip<T>(a, pa, BH, N, dv, c0, w, false, st)) &&
                ok(slice_flip<T>(b, pb, BH, N, dv, c0, w, false, st)) &&
                fwd(pa, pb, c, dec, parts + (size_t)p * nQ, w, dk);
        }
        return r == RET_OK;
    };
    // dQ = forward(dO, V, K), the dv contraction in pieces
    if (P == 1) {
        fwd(dout, v, k, decay, dq, dv, dk);
    } else {
        pieces(dout, v, k, decay);
        if (r == RET_OK) {
            ok(sum_flip<T>(parts, P, nQ, static_cast<T*>(dq), BH, N, dk, false, st));
        }
    }
    // time-reversed copies (and gates reversed and shifted by one)
    if (r == RET_OK) {
        ok(slice_flip<T>(q, Qf, BH, N, dk, 0, dk, true, st)) && ok(slice_flip<T>(k, Kf, BH, N, dk, 0, dk, true, st)) &&
            ok(slice_flip<T>(v, Vf, BH, N, dv, 0, dv, true, st)) && ok(slice_flip<T>(dout, dOf, BH, N, dv, 0, dv, true, st));
        if (GATED && r == RET_OK) {
            gate_flip_kernel<<<grid_for((size_t)BH * N), kBwdThreads, 0, st>>>(decay, gf, N, (size_t)BH * N);
            ok(launch_status());
        }
    }
    const float* dec_rev = GATED ? gf : decay;
    // dK = reverse(forward(rev V, rev dO, rev Q)), in pieces
    if (r == RET_OK) {
        if (P == 1)
            fwd(Vf, dOf, Qf, dec_rev, parts, dv, dk);
        else
            pieces(Vf, dOf, Qf, dec_rev);
    }
    if (r == RET_OK) {
        ok(sum_flip<T>(parts, P, nQ, static_cast<T*>(dk_out), BH, N, dk, true, st));
    }
    // dV = reverse(forward(rev K, rev Q, rev dO))
    if (r == RET_OK && fwd(Kf, Qf, dOf, dec_rev, Rf, dk, dv)) ok(slice_flip<T>(Rf, dv_out, BH, N, dv, 0, dv, true, st));
    // decay gradient
    if (r == RET_OK && ddecay)
        ok(decay_grad<T, GATED>(static_cast<const T*>(q), static_cast<const T*>(dq), static_cast<const T*>(k),
                                static_cast<const T*>(dk_out), decay, ddecay, BH, H, N, dk, st));
    if (cudaFreeAsync(sc, st) != cudaSuccess && r == RET_OK) r = RET_ERR_CUDA;
    return r;
}

template <bool GATED>
ret_status backward_entry(const void* q, const void* k, const void* v, const float* decay, const void* dout, void* dq,
                          void* dk_out, void* dv_out, float* ddecay, int B, int H, int N, int dk, int dv, int chunk,
                          ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (chunk <= 0) return RET_ERR_SHAPE;
    if (dk > 256) return RET_ERR_UNSUPPORTED;
    if (!q || !k || !v || !decay || !dout || !dq || !dk_out || !dv_out) return RET_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    if (N == 0) {
        if (!GATED && ddecay && cudaMemsetAsync(ddecay, 0, sizeof(float) * (size_t)H, st) != cudaSuccess)
            return RET_ERR_CUDA;
        return RET_OK;
    }
    if (dt == RET_BF16) {
        for (const void* p : {q, k, v, dout, static_cast<const void*>(dq), static_cast<const void*>(dk_out),
                              static_cast<const void*>(dv_out)})
            if (!aligned16(p)) return RET_ERR_ALIGN;
        return backward_impl<__nv_bfloat16, GATED>(q, k, v, decay, dout, dq, dk_out, dv_out, ddecay, B, H, N, dk, dv,
                                                   chunk, dt, st);
    }
    return backward_impl<float, GATED>(q, k, v, decay, dout, dq, dk_out, dv_out, ddecay, B, H, N, dk, dv, chunk, dt,
                                       st);
}

// Multi-scale retention output epilogue: the vector kernel when rows are whole 16-byte
// chunks (LPR lanes per row, CH chunks per lane), else the scalar kernel.
template <typename T, int LPR, int CH>
void launch_norm_vec(const T* o, const T* gate, T* y, int H, int N, int dv, float eps, size_t rows, cudaStream_t st) {
    const size_t rows_per_block = (size_t)(kNormThreads / 32) * (32 / LPR);
    const size_t blocks = std::min<size_t>((rows + rows_per_block - 1) / rows_per_block, (size_t)32 * tc::sm_count());
    norm_gate_vec_kernel<T, LPR, CH><<<(unsigned)blocks, kNormThreads, 0, st>>>(o, gate, y, H, N, dv, eps, rows);
}

template <typename T>
ret_status launch_norm_gate(const void* o_, const void* gate_, void* y_, int B, int H, int N, int dv, float eps,
                            cudaStream_t st) {
    const T* o = static_cast<const T*>(o_);
    const T* gate = static_cast<const T*>(gate_);
    T* y = static_cast<T*>(y_);
    const size_t rows = (size_t)B * N * H;
    const bool vec = ((size_t)dv * sizeof(T)) % 16 == 0 && aligned16(o) && aligned16(gate) && aligned16(y);
    const int chunks = vec ? (int)((size_t)dv * sizeof(T) / 16) : 0;
    if (vec && chunks <= 1) launch_norm_vec<T, 1, 1>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 2) launch_norm_vec<T, 2, 1>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 4) launch_norm_vec<T, 4, 1>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 8) launch_norm_vec<T, 8, 1>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 16) launch_norm_vec<T, 16, 1>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 32) launch_norm_vec<T, 32, 1>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 64) launch_norm_vec<T, 32, 2>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 128) launch_norm_vec<T, 32, 4>(o, gate, y, H, N, dv, eps, rows, st);
    else if (vec && chunks <= 256) launch_norm_vec<T, 32, 8>(o, gate, y, H, N, dv, eps, rows, st);
    else {
        const size_t blocks = std::min<size_t>((rows + kNormThreads / 32 - 1) / (kNormThreads / 32),
                                               (size_t)32 * tc::sm_count());
        norm_gate_scalar_kernel<T><<<(unsigned)blocks, kNormThreads, 0, st>>>(o, gate, y, H, N, dv, eps, rows);
    }
    return launch_status();
}

inline bool ranges_overlap(const void* a, const void* b, size_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), z = reinterpret_cast<uintptr_t>(b);
    return x < z + bytes && z < x + bytes;
}

template <typename T>
ret_status launch_parallel(const void* q, const void* k, const void* v, const float* gamma, void* o,
                           int B, int H, int N, int dk, int dv, cudaStream_t st) {
    dim3 grid((N + kParQ - 1) / kParQ, (dv + kParV - 1) / kParV, B * H);
    if (grid.y > (unsigned)kMaxGridY) return RET_ERR_UNSUPPORTED;
    parallel_simt_kernel<T><<<grid, kParThreads, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                          static_cast<const T*>(v), gamma, static_cast<T*>(o),
                                                          H, N, dk, dv);
    return launch_status();
}

template <typename T, bool GATED>
ret_status launch_step(const void* q, const void* k, const void* v, const float* gamma, float* state, void* o,
                       int B, int H, int dk, int dv, cudaStream_t st) {
    const size_t smem = sizeof(float) * 2 * (size_t)dk;
    if ((dv & 3) == 0 && aligned16(state)) {
        const int groups = dv / 4;
        dim3 grid((groups + kDecThreads - 1) / kDecThreads, B * H);
        recurrent_step_vec_kernel<T, GATED><<<grid, kDecThreads, smem, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), gamma, state,
            static_cast<T*>(o), H, dk, dv);
    } else {
        dim3 grid((dv + kDecThreads - 1) / kDecThreads, B * H);
        recurrent_step_scalar_kernel<T, GATED><<<grid, kDecThreads, smem, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), gamma, state,
            static_cast<T*>(o), H, dk, dv);
    }
    return launch_status();
}

// Streams of the host-buffer calls, one set per device with its own mutex (held while a call
// enqueues): cs runs the groups' device work, os their copies out, and the events order them.
// They are separate from the backward's streams, which a host-buffer backward uses inside
// each group.
constexpr int kPipeGroups = 8;
struct HostPipe {
    cudaStream_t cs = nullptr, os = nullptr;
    cudaEvent_t ev[4 + 2 * kPipeGroups] = {};
};
inline std::mutex& pipe_mutex() {
    static std::mutex m;
    return m;
}
inline HostPipe* host_pipe() {
    static HostPipe pipes[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    HostPipe& hp = pipes[dev];
    if (!hp.cs) {  // publish only once every stream and event exists
        HostPipe n;
        bool ok = cudaStreamCreateWithFlags(&n.cs, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&n.os, cudaStreamNonBlocking) == cudaSuccess;
        for (cudaEvent_t& e : n.ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            for (cudaEvent_t e : n.ev)
                if (e) cudaEventDestroy(e);
            if (n.cs) cudaStreamDestroy(n.cs);
            if (n.os) cudaStreamDestroy(n.os);
            return nullptr;
        }
        hp = n;
    }
    return &hp;
}

// The heads of a host-buffer call cut into at most kPipeGroups groups: whole batches when
// B >= kPipeGroups, else runs of heads inside one batch, so that each group is one (B', H')
// problem with its own slice of gamma (heads h0 .. h0 + nh) or of g.
struct HeadGroup {
    int b0, nb, h0, nh;
};
inline int head_groups(int B, int H, HeadGroup (&grp)[kPipeGroups]) {
    int G = 0;
    if (B >= kPipeGroups) {
        const int bpg = (B + kPipeGroups - 1) / kPipeGroups;
        for (int b0 = 0; b0 < B; b0 += bpg) grp[G++] = {b0, std::min(bpg, B - b0), 0, H};
    } else {
        const int per_batch = kPipeGroups / B, hpg = (H + per_batch - 1) / per_batch;
        for (int b = 0; b < B; ++b)
            for (int h0 = 0; h0 < H; h0 += hpg) grp[G++] = {b, 1, h0, std::min(hpg, H - h0)};
    }
    return G;
}

// The chunkwise forward from host buffers: q, k, v, the decay and o live in host memory.
// The heads are cut into head_groups() and pipelined over three streams:
//   st:  fork | H2D of group 0 | H2D of group 1 | ...            | wait cs, os | free
//   cs:        wait H2D g -> chunkwise forward of group g -> ...
//   os:                      wait forward g -> D2H of group g's o -> ...
// so the copies in (the larger part) run back to back while earlier groups compute and copy
// out in the other direction. Device buffers come from the stream-ordered pool. The backward
// from host buffers below follows the same plan.
template <bool GATED>
ret_status chunkwise_host_entry(const void* q, const void* k, const void* v, const float* decay, void* o, int B,
                                int H, int N, int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (chunk <= 0) return RET_ERR_SHAPE;
    if (dk > 256) return RET_ERR_UNSUPPORTED;
    if (N == 0) return RET_OK;
    if (!q || !k || !v || !decay || !o) return RET_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    const size_t es = dt == RET_F32 ? 4 : 2;
    const size_t head_q = (size_t)N * dk * es, head_v = (size_t)N * dv * es, head_g = (size_t)N * sizeof(float);
    const size_t BH = (size_t)B * H;
    const size_t sz[5] = {BH * head_q, BH * head_q, BH * head_v, BH * head_v,
                          GATED ? BH * head_g : (size_t)H * sizeof(float)};
    size_t off[5], bytes = 0;
    for (int i = 0; i < 5; ++i) {
        off[i] = bytes;
        bytes += align256(sz[i]);
    }
    HeadGroup grp[kPipeGroups];
    const int G = head_groups(B, H, grp);
    std::lock_guard<std::mutex> lock(pipe_mutex());
    HostPipe* hp = host_pipe();
    if (!hp) return RET_ERR_CUDA;
    cudaStream_t cs = hp->cs, os = hp->os;
    cudaEvent_t ev_fork = hp->ev[0], ev_cs = hp->ev[1], ev_os = hp->ev[2];
    cudaEvent_t* ev_in = hp->ev + 4;                 // [kPipeGroups]: group g's inputs are on the device
    cudaEvent_t* ev_out = hp->ev + 4 + kPipeGroups;  // [kPipeGroups]: group g's results are computed
    tc::keep_pool_memory();
    uint8_t* buf = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void**>(&buf), bytes, st) != cudaSuccess) return RET_ERR_CUDA;
    uint8_t* dq = buf + off[0];
    uint8_t* dk_ = buf + off[1];
    uint8_t* dv_ = buf + off[2];
    uint8_t* do_ = buf + off[3];
    float* ddec = reinterpret_cast<float*>(buf + off[4]);
    const uint8_t* hq = static_cast<const uint8_t*>(q);
    const uint8_t* hk = static_cast<const uint8_t*>(k);
    const uint8_t* hv = static_cast<const uint8_t*>(v);
    uint8_t* ho = static_cast<uint8_t*>(o);
    ret_status r = RET_OK;
    auto cu = [&](cudaError_t e) {
        if (r == RET_OK && e != cudaSuccess) r = RET_ERR_CUDA;
        return r == RET_OK;
    };
    auto h2d = [&](void* d, const void* h, size_t n) { return cu(cudaMemcpyAsync(d, h, n, cudaMemcpyHostToDevice, st)); };
    if (!GATED) h2d(ddec, decay, sz[4]);
    if (cu(cudaEventRecord(ev_fork, st))) {
        cu(cudaStreamWaitEvent(cs, ev_fork, 0));
        cu(cudaStreamWaitEvent(os, ev_fork, 0));
    }
    for (int gi = 0; gi < G && r == RET_OK; ++gi) {
        const HeadGroup& g = grp[gi];
        const size_t first = (size_t)g.b0 * H + g.h0, heads = (size_t)g.nb * g.nh;
        h2d(dq + first * head_q, hq + first * head_q, heads * head_q);
        h2d(dk_ + first * head_q, hk + first * head_q, heads * head_q);
        h2d(dv_ + first * head_v, hv + first * head_v, heads * head_v);
        if (GATED)
            h2d(reinterpret_cast<uint8_t*>(ddec) + first * head_g, reinterpret_cast<const uint8_t*>(decay) +
                first * head_g, heads * head_g);
        if (!cu(cudaEventRecord(ev_in[gi], st)) || !cu(cudaStreamWaitEvent(cs, ev_in[gi], 0))) break;
        const float* gdec = GATED ? ddec + first * N : ddec + g.h0;
        const ret_status rc = chunkwise_entry<GATED>(dq + first * head_q, dk_ + first * head_q, dv_ + first * head_v,
                                                     gdec, do_ + first * head_v, nullptr, nullptr, g.nb, g.nh, N, dk,
                                                     dv, chunk, dt, cs);
        if (rc != RET_OK && r == RET_OK) r = rc;
        if (!cu(cudaEventRecord(ev_out[gi], cs)) || !cu(cudaStreamWaitEvent(os, ev_out[gi], 0))) break;
        cu(cudaMemcpyAsync(ho + first * head_v, do_ + first * head_v, heads * head_v, cudaMemcpyDeviceToHost, os));
    }
    // join both library streams back into st whatever happened, then release the buffers
    const bool joined = cudaEventRecord(ev_cs, cs) == cudaSuccess && cudaEventRecord(ev_os, os) == cudaSuccess &&
                        cudaStreamWaitEvent(st, ev_cs, 0) == cudaSuccess &&
                        cudaStreamWaitEvent(st, ev_os, 0) == cudaSuccess;
    if (!joined) {
        cudaStreamSynchronize(cs);
        cudaStreamSynchronize(os);
        if (r == RET_OK) r = RET_ERR_CUDA;
    }
    if (cudaFreeAsync(buf, st) != cudaSuccess && r == RET_OK) r = RET_ERR_CUDA;
    return r;
}

// The backward from host buffers: q, k, v, the decay and dO in host memory, dq, dk, dv and
// the decay gradient written back to host memory. Same plan as chunkwise_host_entry: the
// copies in run back to back on st; cs runs each group's backward (the device-buffer call,
// with its own library streams) once its inputs have landed; os copies its gradients out.
// Each group's arrays start on 256-byte boundaries of the device buffers. dgamma sums over
// batches and tokens, so each group writes its heads' share into a row of its own
// (zeroed first, [G, H]) and one small kernel adds the rows once every group is done.
template <bool GATED>
ret_status backward_host_entry(const void* q, const void* k, const void* v, const float* decay, const void* dout,
                               void* dq, void* dk_out, void* dv_out, float* ddecay, int B, int H, int N, int dk,
                               int dv, int chunk, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (chunk <= 0) return RET_ERR_SHAPE;
    if (dk > 256) return RET_ERR_UNSUPPORTED;
    if (!q || !k || !v || !decay || !dout || !dq || !dk_out || !dv_out) return RET_ERR_NULL;
    if (N == 0) {
        if (!GATED && ddecay) std::memset(ddecay, 0, sizeof(float) * (size_t)H);
        return RET_OK;
    }
    cudaStream_t st = as_stream(stream);
    const size_t es = dt == RET_F32 ? 4 : 2;
    const size_t head_q = (size_t)N * dk * es, head_v = (size_t)N * dv * es, head_g = (size_t)N * sizeof(float);
    HeadGroup grp[kPipeGroups];
    const int G = head_groups(B, H, grp);
    // per array, each group's region from a 256-byte boundary
    size_t goff[kPipeGroups + 1][3] = {};  // [group][q-like, v-like, per-token fp32]
    for (int gi = 0; gi < G; ++gi) {
        const size_t heads = (size_t)grp[gi].nb * grp[gi].nh;
        goff[gi + 1][0] = goff[gi][0] + align256(heads * head_q);
        goff[gi + 1][1] = goff[gi][1] + align256(heads * head_v);
        goff[gi + 1][2] = goff[gi][2] + align256(heads * head_g);
    }
    const size_t QB = goff[G][0], VB = goff[G][1], GB = goff[G][2];
    // q, k, dq, dk | v, dO, dv | g, dg (gated) or gamma, dgamma rows and sum (fixed)
    const size_t fixed_bytes = align256(sizeof(float) * H) * 2 + align256(sizeof(float) * (size_t)G * H);
    const size_t bytes = 4 * QB + 3 * VB + (GATED ? 2 * GB : fixed_bytes);
    std::lock_guard<std::mutex> lock(pipe_mutex());
    HostPipe* hp = host_pipe();
    if (!hp) return RET_ERR_CUDA;
    cudaStream_t cs = hp->cs, os = hp->os;
    cudaEvent_t ev_fork = hp->ev[0], ev_cs = hp->ev[1], ev_os = hp->ev[2], ev_sum = hp->ev[3];
    cudaEvent_t* ev_in = hp->ev + 4;
    cudaEvent_t* ev_out = hp->ev + 4 + kPipeGroups;
    tc::keep_pool_memory();
    uint8_t* buf = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void**>(&buf), bytes, st) != cudaSuccess) return RET_ERR_CUDA;
    uint8_t* d_q = buf;
    uint8_t* d_k = d_q + QB;
    uint8_t* d_dq = d_k + QB;
    uint8_t* d_dk = d_dq + QB;
    uint8_t* d_v = d_dk + QB;
    uint8_t* d_do = d_v + VB;
    uint8_t* d_dv = d_do + VB;
    uint8_t* d_g = d_dv + VB;                       // gated: g, then dg
    uint8_t* d_dg = d_g + GB;
    float* d_gamma = reinterpret_cast<float*>(d_g);  // fixed: gamma [H], dgamma rows [G, H], dgamma [H]
    float* d_rows = reinterpret_cast<float*>(d_g + align256(sizeof(float) * H));
    float* d_dgamma = reinterpret_cast<float*>(d_g + align256(sizeof(float) * H) + align256(sizeof(float) * (size_t)G * H));
    ret_status r = RET_OK;
    auto cu = [&](cudaError_t e) {
        if (r == RET_OK && e != cudaSuccess) r = RET_ERR_CUDA;
        return r == RET_OK;
    };
    auto h2d = [&](void* d, const void* h, size_t n) { return cu(cudaMemcpyAsync(d, h, n, cudaMemcpyHostToDevice, st)); };
    auto d2h = [&](void* h, const void* d, size_t n) { return cu(cudaMemcpyAsync(h, d, n, cudaMemcpyDeviceToHost, os)); };
    const bool want_dgamma = !GATED && ddecay;
    if (!GATED) h2d(d_gamma, decay, sizeof(float) * H);
    if (want_dgamma) cu(cudaMemsetAsync(d_rows, 0, sizeof(float) * (size_t)G * H, st));
    if (cu(cudaEventRecord(ev_fork, st))) {
        cu(cudaStreamWaitEvent(cs, ev_fork, 0));
        cu(cudaStreamWaitEvent(os, ev_fork, 0));
    }
    for (int gi = 0; gi < G && r == RET_OK; ++gi) {
        const HeadGroup& g = grp[gi];
        const size_t first = (size_t)g.b0 * H + g.h0, heads = (size_t)g.nb * g.nh;
        const size_t oq = goff[gi][0], ov = goff[gi][1], og = goff[gi][2];
        h2d(d_q + oq, static_cast<const uint8_t*>(q) + first * head_q, heads * head_q);
        h2d(d_k + oq, static_cast<const uint8_t*>(k) + first * head_q, heads * head_q);
        h2d(d_v + ov, static_cast<const uint8_t*>(v) + first * head_v, heads * head_v);
        h2d(d_do + ov, static_cast<const uint8_t*>(dout) + first * head_v, heads * head_v);
        if (GATED) h2d(d_g + og, reinterpret_cast<const uint8_t*>(decay) + first * head_g, heads * head_g);
        if (!cu(cudaEventRecord(ev_in[gi], st)) || !cu(cudaStreamWaitEvent(cs, ev_in[gi], 0))) break;
        const float* gdec = GATED ? reinterpret_cast<const float*>(d_g + og) : d_gamma + g.h0;
        float* gdd = GATED ? (ddecay ? reinterpret_cast<float*>(d_dg + og) : nullptr)
                           : (want_dgamma ? d_rows + (size_t)gi * H + g.h0 : nullptr);
        const ret_status rc = backward_entry<GATED>(d_q + oq, d_k + oq, d_v + ov, gdec, d_do + ov, d_dq + oq, d_dk + oq,
                                                    d_dv + ov, gdd, g.nb, g.nh, N, dk, dv, chunk, dt, cs);
        if (rc != RET_OK && r == RET_OK) r = rc;
        if (!cu(cudaEventRecord(ev_out[gi], cs)) || !cu(cudaStreamWaitEvent(os, ev_out[gi], 0))) break;
        d2h(static_cast<uint8_t*>(dq) + first * head_q, d_dq + oq, heads * head_q);
        d2h(static_cast<uint8_t*>(dk_out) + first * head_q, d_dk + oq, heads * head_q);
        d2h(static_cast<uint8_t*>(dv_out) + first * head_v, d_dv + ov, heads * head_v);
        if (GATED && ddecay) d2h(reinterpret_cast<uint8_t*>(ddecay) + first * head_g, d_dg + og, heads * head_g);
    }
    if (want_dgamma && r == RET_OK) {
        sum_rows_kernel<<<(H + kBwdThreads - 1) / kBwdThreads, kBwdThreads, 0, cs>>>(d_rows, G, H, d_dgamma);
        if (cu(cudaGetLastError()) && cu(cudaEventRecord(ev_sum, cs)) && cu(cudaStreamWaitEvent(os, ev_sum, 0)))
            d2h(ddecay, d_dgamma, sizeof(float) * H);
    }
    const bool joined = cudaEventRecord(ev_cs, cs) == cudaSuccess && cudaEventRecord(ev_os, os) == cudaSuccess &&
                        cudaStreamWaitEvent(st, ev_cs, 0) == cudaSuccess &&
                        cudaStreamWaitEvent(st, ev_os, 0) == cudaSuccess;
    if (!joined) {
        cudaStreamSynchronize(cs);
        cudaStreamSynchronize(os);
        if (r == RET_OK) r = RET_ERR_CUDA;
    }
    if (cudaFreeAsync(buf, st) != cudaSuccess && r == RET_OK) r = RET_ERR_CUDA;
    return r;
}

}  // namespace

extern "C" {

ret_status ret_parallel(const void* q, const void* k, const void* v, const float* gamma, void* o,
                        int B, int H, int N, int dk, int dv, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (dk > 1024) return RET_ERR_UNSUPPORTED;
    if (N == 0) return RET_OK;
    if (!q || !k || !v || !gamma || !o) return RET_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    return dt == RET_F32 ? launch_parallel<float>(q, k, v, gamma, o, B, H, N, dk, dv, st)
                         : launch_parallel<__nv_bfloat16>(q, k, v, gamma, o, B, H, N, dk, dv, st);
}

ret_status ret_chunkwise(const void* q, const void* k, const void* v, const float* gamma, void* o,
                         const float* state_in, float* state_out, int B, int H, int N, int dk, int dv,
                         int chunk, ret_dtype dt, void* stream) {
    return chunkwise_entry<false>(q, k, v, gamma, o, state_in, state_out, B, H, N, dk, dv, chunk, dt, stream);
}

ret_status gated_ret_chunkwise(const void* q, const void* k, const void* v, const float* g, void* o,
                               const float* state_in, float* state_out, int B, int H, int N, int dk, int dv,
                               int chunk, ret_dtype dt, void* stream) {
    return chunkwise_entry<true>(q, k, v, g, o, state_in, state_out, B, H, N, dk, dv, chunk, dt, stream);
}

ret_status ret_chunkwise_host(const void* q, const void* k, const void* v, const float* gamma, void* o, int B, int H,
                              int N, int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    return chunkwise_host_entry<false>(q, k, v, gamma, o, B, H, N, dk, dv, chunk, dt, stream);
}

ret_status gated_ret_chunkwise_host(const void* q, const void* k, const void* v, const float* g, void* o, int B,
                                    int H, int N, int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    return chunkwise_host_entry<true>(q, k, v, g, o, B, H, N, dk, dv, chunk, dt, stream);
}

ret_status ret_recurrent_step(const void* q, const void* k, const void* v, const float* gamma, float* state,
                              void* o, int B, int H, int dk, int dv, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, 1, dk, dv, dt);
    if (s != RET_OK) return s;
    if (dk > 4096) return RET_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gamma || !state || !o) return RET_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    return dt == RET_F32 ? launch_step<float, false>(q, k, v, gamma, state, o, B, H, dk, dv, st)
                         : launch_step<__nv_bfloat16, false>(q, k, v, gamma, state, o, B, H, dk, dv, st);
}

ret_status gated_ret_recurrent_step(const void* q, const void* k, const void* v, const float* g, float* state,
                                    void* o, int B, int H, int dk, int dv, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, 1, dk, dv, dt);
    if (s != RET_OK) return s;
    if (dk > 4096) return RET_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !state || !o) return RET_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    return dt == RET_F32 ? launch_step<float, true>(q, k, v, g, state, o, B, H, dk, dv, st)
                         : launch_step<__nv_bfloat16, true>(q, k, v, g, state, o, B, H, dk, dv, st);
}

const char* ret_status_str(ret_status s) {
    switch (s) {
        case RET_OK: return "ok";
        case RET_ERR_NULL: return "a required pointer is NULL";
        case RET_ERR_SHAPE: return "invalid size";
        case RET_ERR_DTYPE: return "invalid dtype";
        case RET_ERR_UNSUPPORTED: return "sizes not supported by the kernels";
        case RET_ERR_CUDA: return "CUDA error";
        case RET_ERR_TIMEOUT: return "a kernel wait timed out (device error word set)";
        case RET_ERR_ALIGN: return "pointer not 16-byte aligned";
        case RET_ERR_SCRATCH: return "problem needs more scratch than the fixed no-allocation buffer holds";
    }
    return "unknown status";
}

ret_status ret_last_device_error(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return RET_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return RET_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return RET_ERR_CUDA;
    return word ? RET_ERR_TIMEOUT : RET_OK;
}

int ret_chunkwise_path(int dk, int dv, int chunk, ret_dtype dt) {
    if ((dt != RET_F32 && dt != RET_BF16) || dk <= 0 || dv <= 0 || chunk <= 0 || dk > 256) return -1;
    return tc_chunk_supported(dk, dv, chunk, dt == RET_BF16) ? 1 : 0;
}

int ret_chunkwise_launches(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt) {
    if (check_common(B, H, N, dk, dv, dt) != RET_OK || chunk <= 0 || dk > 256) return -1;
    if (N == 0) return 0;
    if (tc_chunk_supported(dk, dv, chunk, dt == RET_BF16)) return tc_chunk_launches(B, H, N, dk, dv);
    return 1;
}

ret_status ret_chunkwise_state(const void* k, const void* v, const float* gamma, float* state_out, float* log2_decay,
                               int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    return chunkwise_state_entry<false>(k, v, gamma, state_out, log2_decay, B, H, N, dk, dv, chunk, dt, stream);
}

ret_status gated_ret_chunkwise_state(const void* k, const void* v, const float* g, float* state_out,
                                     float* log2_decay, int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt,
                                     void* stream) {
    return chunkwise_state_entry<true>(k, v, g, state_out, log2_decay, B, H, N, dk, dv, chunk, dt, stream);
}

ret_status ret_state_prefix(const float* seg_states, const float* seg_log2_decay, const float* state_in,
                            float* start_states, float* end_state, int R, int B, int H, int dk, int dv, void* stream) {
    if (R <= 0 || B <= 0 || H <= 0 || dk <= 0 || dv <= 0) return RET_ERR_SHAPE;
    if (!seg_states || !seg_log2_decay || !start_states) return RET_ERR_NULL;
    const long long n = (long long)B * H * dk * dv;
    if ((long long)dk * dv > 0x7fffffffLL) return RET_ERR_UNSUPPORTED;
    const int blocks = (int)std::min<long long>((n + 255) / 256, 4LL * tc::sm_count());
    state_prefix_kernel<<<blocks, 256, 0, as_stream(stream)>>>(seg_states, seg_log2_decay, state_in, start_states,
                                                                end_state, R, B * H, dk * dv);
    return launch_status();
}

ret_status ret_selftest_wait_timeout(unsigned int limit_us, void* stream) {
    if (limit_us == 0 || limit_us > 1000000u) return RET_ERR_SHAPE;
    if (!tc::tc_device_ok()) return RET_ERR_UNSUPPORTED;
    tc::selftest_wait_kernel<<<1, 64, 0, as_stream(stream)>>>((unsigned long long)limit_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? RET_OK : RET_ERR_CUDA;
}

ret_status ret_chunkwise_backward(const void* q, const void* k, const void* v, const float* gamma, const void* dout,
                                  void* dq, void* dk, void* dv, float* dgamma, int B, int H, int N, int dk_dim,
                                  int dv_dim, int chunk, ret_dtype dt, void* stream) {
    return backward_entry<false>(q, k, v, gamma, dout, dq, dk, dv, dgamma, B, H, N, dk_dim, dv_dim, chunk, dt, stream);
}

ret_status gated_ret_chunkwise_backward(const void* q, const void* k, const void* v, const float* g, const void* dout,
                                        void* dq, void* dk, void* dv, float* dg, int B, int H, int N, int dk_dim,
                                        int dv_dim, int chunk, ret_dtype dt, void* stream) {
    return backward_entry<true>(q, k, v, g, dout, dq, dk, dv, dg, B, H, N, dk_dim, dv_dim, chunk, dt, stream);
}

ret_status ret_chunkwise_backward_host(const void* q, const void* k, const void* v, const float* gamma,
                                       const void* dout, void* dq, void* dk, void* dv, float* dgamma, int B, int H,
                                       int N, int dk_dim, int dv_dim, int chunk, ret_dtype dt, void* stream) {
    return backward_host_entry<false>(q, k, v, gamma, dout, dq, dk, dv, dgamma, B, H, N, dk_dim, dv_dim, chunk, dt,
                                      stream);
}

ret_status gated_ret_chunkwise_backward_host(const void* q, const void* k, const void* v, const float* g,
                                             const void* dout, void* dq, void* dk, void* dv, float* dg, int B, int H,
                                             int N, int dk_dim, int dv_dim, int chunk, ret_dtype dt, void* stream) {
    return backward_host_entry<true>(q, k, v, g, dout, dq, dk, dv, dg, B, H, N, dk_dim, dv_dim, chunk, dt, stream);
}

int ret_chunkwise_state_launches(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt) {
    if (check_common(B, H, N, dk, dv, dt) != RET_OK || chunk <= 0 || dk > 256) return -1;
    if (N == 0) return 0;
    // the decay kernel, then the state-only pass (+ prefix) or the CUDA-core chunkwise kernel
    return 1 + (tc_chunk_supported(dk, dv, chunk, dt == RET_BF16) ? tc_state_launches(B, H, N, dv) : 1);
}

ret_status ret_msr_norm_gate(const void* o, const void* gate, void* y, int B, int H, int N, int dv, float eps,
                             ret_dtype dt, void* stream) {
    if (dt != RET_F32 && dt != RET_BF16) return RET_ERR_DTYPE;
    // the kernels stride over rows, so B * H has no grid limit here
    if (B <= 0 || H <= 0 || N < 0 || dv <= 0) return RET_ERR_SHAPE;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return RET_ERR_SHAPE;
    if (N == 0) return RET_OK;
    if (!o || !gate || !y) return RET_ERR_NULL;
    const size_t bytes = (size_t)B * H * N * dv * (dt == RET_BF16 ? 2 : 4);
    // y may be the gate buffer itself; any other overlap would race
    if (ranges_overlap(y, o, bytes) || (y != gate && ranges_overlap(y, gate, bytes))) return RET_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (dt == RET_BF16) return launch_norm_gate<__nv_bfloat16>(o, gate, y, B, H, N, dv, eps, st);
    return launch_norm_gate<float>(o, gate, y, B, H, N, dv, eps, st);
}

int ret_chunkwise_backward_launches(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt, int gated,
                                    int ddecay) {
    if (check_common(B, H, N, dk, dv, dt) != RET_OK || chunk <= 0 || dk > 256) return -1;
    if (N == 0) return 0;
    if (backward_on_tensor_cores(dk, dv, chunk, dt)) return backward_tc_launches(B, H, N, dk, dv, gated, ddecay);
    // mirrors backward_impl's copying path: forward calls, the slice / flip / sum kernels, the decay gradient
    auto fwd = [&](int wq, int wv) { return ret_chunkwise_launches(B, H, N, wq, wv, chunk, dt); };
    const int pw = dv <= 256 ? dv : 256, P = (dv + pw - 1) / pw;
    int n = 0;
    for (int p = 0; p < P; ++p) {
        const int w = std::min(pw, dv - p * pw);
        // two slices, then the forward, for a dQ and a dK piece
        n += P == 1 ? 2 * fwd(dv, dk) : 2 * (2 + fwd(w, dk));
    }
    n += P == 1 ? 0 : 1;                 // sum of the dQ pieces
    n += 4 + (gated ? 1 : 0);            // reversed Q, K, V, dO (and gates)
    n += 1;                              // sum + flip of the dK pieces
    n += fwd(dk, dv) + 1;                // dV and its flip
    n += ddecay ? (gated ? 2 : 1) : 0;   // decay gradient (gated: and its suffix sum)
    return n;
}

const char* ret_version(void) { return "0.1.0"; }

}  // extern "C"

// ------------------------------------------------------------------ no-allocation entry point
//
// For callers that must not let the library allocate device memory (their own
// allocator owns the memory, or allocation is forbidden after start-up): the
// scratch of a split sequence comes from this fixed buffer instead of the
// stream-ordered pool. Each device that loads the library holds the buffer
// until exit. Host code must not use its name as a pointer (that is a
// host-side stand-in); the device address is looked up once per device below.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[RET_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device, looked up on the
// first call per device (with that device current) and cached; null on error.
void* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

// The segment plan of a no-allocation call: ret_chunkwise's, or, when that does not fit
// the fixed buffer, one state-only piece per segment (less scratch, same result up to
// rounding order).
tc::Plan noalloc_plan(int B, int H, int N, int dk, int dv, bool alias) {
    tc::Plan pl = tc::plan(B, H, N, dv);
    if (tc::scratch_bytes(pl, B * H, dk, dv, alias) > RET_NOALLOC_SCRATCH_BYTES) pl = tc::plan(B, H, N, dv, false);
    return pl;
}

}  // namespace

extern "C" long long ret_chunkwise_noalloc_scratch_bytes(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt,
                                                         int in_place) {
    if (check_common(B, H, N, dk, dv, dt) != RET_OK || chunk <= 0 || dk > 256) return -1;
    if (N == 0 || !tc_chunk_supported(dk, dv, chunk, dt == RET_BF16)) return 0;
    const tc::Plan pl = noalloc_plan(B, H, N, dk, dv, in_place != 0);
    return (long long)tc::scratch_bytes(pl, B * H, dk, dv, in_place != 0);
}

extern "C" ret_status ret_chunkwise_noalloc(const void* q, const void* k, const void* v, const float* gamma,
                                            void* o, const float* state_in, float* state_out, int B, int H, int N,
                                            int dk, int dv, int chunk, ret_dtype dt, void* stream) {
    ret_status s = check_common(B, H, N, dk, dv, dt);
    if (s != RET_OK) return s;
    if (chunk <= 0) return RET_ERR_SHAPE;
    if (dk > 256) return RET_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (N == 0) return empty_sequence_state(state_in, state_out, B, H, dk, dv, st);  // copy or memset only
    if (!q || !k || !v || !gamma || !o) return RET_ERR_NULL;
    if (!tc_chunk_supported(dk, dv, chunk, dt == RET_BF16)) {
        // the CUDA-core kernel keeps its state in shared memory and needs no scratch
        return dt == RET_F32 ? launch_chunkwise_simt<float, false>(q, k, v, gamma, o, state_in, state_out, B, H, N,
                                                                   dk, dv, chunk, st)
                             : launch_chunkwise_simt<__nv_bfloat16, false>(q, k, v, gamma, o, state_in, state_out,
                                                                           B, H, N, dk, dv, chunk, st);
    }
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RET_ERR_ALIGN;
    const bool alias = state_in != nullptr && state_in == state_out;
    const tc::Plan pl = noalloc_plan(B, H, N, dk, dv, alias);
    const size_t bytes = tc::scratch_bytes(pl, B * H, dk, dv, alias);
    if (bytes > RET_NOALLOC_SCRATCH_BYTES) return RET_ERR_SCRATCH;
    void* scratch = nullptr;
    if (bytes) {
        scratch = noalloc_scratch();
        if (scratch == nullptr) return RET_ERR_CUDA;
    }
    return tc::launch_with_scratch<false>(q, k, v, gamma, o, state_in, state_out, B, H, N, dk, dv, pl, scratch, st);
}
