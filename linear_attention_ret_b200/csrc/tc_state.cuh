// State-only pass of a split sequence (sm_100a): the end state of each sub-segment from a
// zero start and its total decay, without outputs. Included by tc_chunk.cuh.
//
// Method: "RetNet retention mechanism" (aiqz.cc), section 块级循环 (the state carried
// between chunks, S_i = decay_i S_{i-1} + K_i^T diag(zeta) V_i), and the Gated RetNet
// page's cross_chunk update with per-token decays. Only the update product runs here:
//   S^T += (zeta V / kappa)^T K     M = 128 (dv slice)  N = dk  K = TT tokens   (SS, both MN-major)
// over tiles of TT tokens, with the state held as S = kappa T (T in TMEM, the scalar kappa in
// registers; T is rescaled in place only when kappa would fall below 2^-40).
//
// Roles (192 threads): warp 0 issues the TMA loads (a ring of stages of a K tile and a V
// tile, 192 KB in all: the pass is bound by how fast copies arrive, so it keeps many in
// flight), warp 1 allocates TMEM and issues the products, warps 2-5 turn each V tile into
// zeta V / kappa in place and finally write kappa T. Tiles are 64 tokens for a fixed decay
// (four stages at dk = 256: more copies in flight) and 128 tokens for the gated form, whose
// per-tile work (a scan of the gates, exponentials, more frequent rescaling) is better
// amortised over longer tiles; its gates are copied asynchronously into a shared-memory ring
// kGateTiles tiles ahead, since their latency exceeds a tile's work. REV visits the tiles from the last back with the reversed
// direction's key weights (see chunk_tc_kernel). All waits are bounded like the other
// bodies'.
#pragma once

namespace ret {
namespace tc {

constexpr int kSThreads = 192;
constexpr int kMaxSStages = 8;
constexpr int kGateTiles = 4;  // gated: tiles of gates in flight ahead of the scan

// 4-byte asynchronous copy global -> shared (zero-filled when bytes == 0), its group commit
// and the wait for all but the newest n groups.
__device__ __forceinline__ void cp_async4(float* dst, const float* src, int bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// tokens per tile of the state-only pass
__host__ __device__ constexpr int state_tile(bool gated) { return gated ? 128 : 64; }

template <int DK, int TT>
struct StateLayout {
    static constexpr int kRowBlk = TT * 128;                    // one TT-row x 64-column block (128-byte rows)
    static constexpr int kKBytes = DK / 64 * kRowBlk;           // TT token rows x DK
    static constexpr int kVBytes = 2 * kRowBlk;                 // TT token rows x 128 dv
    static constexpr int kStageBytes = kKBytes + kVBytes;
    static constexpr int kStages = std::min(kMaxSStages, 192 * 1024 / kStageBytes);
    static constexpr int kBar = kStages * kStageBytes;
    static constexpr int kNumBars = 4 * kStages + 1;            // full, empty, zv, upd per stage; drain
    static constexpr int kTab = kBar + kNumBars * 8;            // zeta / kappa [TT], gated cumsum [TT]
    static constexpr int kGRing = kTab + 2 * TT * 4;            // gated: raw gates of kGateTiles tiles
    static constexpr int kTmemSlot = kGRing + kGateTiles * TT * 4;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kSmemAlloc = kBytes + 1024;            // slack to align the base to 1024 B
    static constexpr int kTmemCols = DK <= 32 ? 32 : DK <= 64 ? 64 : DK <= 128 ? 128 : 256;
    static_assert(kSmemAlloc <= 227 * 1024, "shared memory overflow");
};

// Inclusive cumulative sum over 128 values in log2 units by one warp: lane l holds
// x[4l .. 4l+3]; writes cum[0..127].
__device__ __forceinline__ void warp_cumsum128(const float (&x)[4], int lane, float* cum) {
    const float p1 = x[0] + x[1], p2 = p1 + x[2], p3 = p2 + x[3];
    float incl = p3;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const float excl = incl - p3;
    cum[4 * lane] = excl + x[0];
    cum[4 * lane + 1] = excl + p1;
    cum[4 * lane + 2] = excl + p2;
    cum[4 * lane + 3] = excl + p3;
}

// upd[s]: the update of a tile in stage s has completed. One per stage, like the others, so
// that a wait for a given tile's update is never more than one phase behind: the epilogue
// waits on it only now and then (renormalisation, the end), and a single barrier could by
// then have completed two phases, which a parity wait cannot tell from none.
// barrier index of (kind, stage) for NS stages
__host__ __device__ constexpr int sbar(int kind, int stage, int ns) { return kind * ns + stage; }
enum StateBarKind { sFull = 0, sEmpty = 1, sZV = 2, sUpd = 3 };

// Grid: (dv / 128, B*H, sub-segments). p.seg_chunks: 64-token chunks per sub-segment;
// p.units: sub-segments the whole sequence is cut into (REV counts them from the end).
// Writes sub-segment z's end state to seg_state[z] and log2 of its total decay to
// seg_ldec[z].
template <int DK, bool GATED, bool REV>
__global__ void __launch_bounds__(kSThreads, 1)
state_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Params p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int kST = state_tile(GATED);
    using Lay = StateLayout<DK, kST>;
    constexpr int NS = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int b) { return sbase + Lay::kBar + 8 * b; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::kTmemSlot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.x, bh = blockIdx.y, seg = blockIdx.z;
    const int dv0 = slice * kDvS;
    const int tseg = REV ? p.units - 1 - seg : seg;
    const int tbeg = tseg * p.seg_chunks * kC;
    const int tend = min(tbeg + p.seg_chunks * kC, p.N);
    const int ntiles = tend > tbeg ? (tend - tbeg + kST - 1) / kST : 0;
    float* so = p.seg_state + ((size_t)seg * gridDim.y + bh) * DK * p.dv + dv0;
    if (ntiles == 0) {
        // REV only: a sub-segment past the end of a short last segment: zero state, no decay
        for (int e = threadIdx.x; e < DK * kDvS; e += blockDim.x) so[(size_t)(e / kDvS) * p.dv + e % kDvS] = 0.f;
        if (slice == 0 && threadIdx.x == 0) p.seg_ldec[(size_t)seg * gridDim.y + bh] = 0.f;
        return;
    }
    auto tile_t0 = [&](int c) { return tbeg + (REV ? ntiles - 1 - c : c) * kST; };
    auto tile_len = [&](int c) { return min(kST, tend - tile_t0(c)); };

    if (threadIdx.x == 0) {
        for (int b = 0; b < Lay::kNumBars; ++b) mbar_init(bar(b), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(Lay::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = -1;
            for (int c = 0; c < ntiles; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(bar(sbar(sEmpty, s, NS)), ((c / NS) - 1) & 1, abort_flag)) break;
                const uint32_t st = sbase + s * Lay::kStageBytes;
                const int t0 = tile_t0(c);
                const uint32_t fb = bar(sbar(sFull, s, NS));
                mbar_expect_tx(fb, Lay::kStageBytes);
#pragma unroll
                for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                    for (int h = 0; h < kST / 64; ++h)
                        tma_load_3d(st + kb * Lay::kRowBlk + h * kTile64, &tm_k, kb * 64, t0 + 64 * h, bh, fb);
#pragma unroll
                for (int db = 0; db < 2; ++db)
#pragma unroll
                    for (int h = 0; h < kST / 64; ++h)
                        tma_load_3d(st + Lay::kKBytes + db * Lay::kRowBlk + h * kTile64, &tm_v, dv0 + 64 * db,
                                    t0 + 64 * h, bh, fb);
                issued = c;
            }
            if (*abort_flag && issued >= 0) {
                // drain the copies in flight before the CTA may exit
                for (int c = std::max(issued - NS + 1, 0); c <= issued; ++c)
                    mbar_drain(bar(sbar(sFull, c % NS, NS)), (c / NS) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_up = idesc(128, DK, 1, 1);
            for (int c = 0; c < ntiles; ++c) {
                const int s = c % NS;
                const uint32_t sK = sbase + s * Lay::kStageBytes, sZ = sK + Lay::kKBytes;
                if (!mbar_wait(bar(sbar(sFull, s, NS)), (c / NS) & 1, abort_flag) ||
                    !mbar_wait(bar(sbar(sZV, s, NS)), (c / NS) & 1, abort_flag))
                    break;
                tc_fence_after();
                // S^T += (zeta V / kappa)^T K: A = the scaled V tile MN-major (dv blocks kRowBlk apart),
                // B = K tile MN-major (dk blocks kRowBlk apart), 16 tokens per step
#pragma unroll
                for (int ks = 0; ks < kST / 16; ++ks)
                    mma_ss(tmem, sdesc(sZ + ks * 2048, Lay::kRowBlk, 1024), sdesc(sK + ks * 2048, Lay::kRowBlk, 1024),
                           id_up, (c > 0 || ks > 0) ? 1u : 0u);
                mma_commit(bar(sbar(sEmpty, s, NS)));
                mma_commit(bar(sbar(sUpd, s, NS)));
            }
            mma_commit(bar(4 * NS));
            mbar_drain(bar(4 * NS), 0);
        }
    } else {
        // ------------------------------------------------------------ state epilogue (warps 2..5)
        const int ts = threadIdx.x - 64;  // 0..127
        const int quarter = warp & 3;     // TMEM lane quarter this warp may access
        const int d = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float* zk = reinterpret_cast<float*>(sm + Lay::kTab);   // zeta_m / kappa of the current tile
        float* cum = zk + kST;                                   // gated: in-tile cumulative log2 decay
        auto wait_all = [&](int b, uint32_t parity) {
            mbar_wait(bar(b), parity, abort_flag);
            asm volatile("bar.sync 1, 128;" ::: "memory");
            return *abort_flag == 0;
        };
        const float lg = GATED ? 0.f : log2f(p.decay_in[bh % p.H]);
        const float* G = GATED ? p.decay_in + (size_t)bh * p.N : nullptr;
        // gated: warp 2 copies the raw gates of tile c into ring slot c % kGateTiles with
        // asynchronous 4-byte copies (lane l: tokens GPL l .. GPL l + GPL - 1, zeros past the
        // tile), kGateTiles tiles ahead of the scan, one commit group per tile, so the scan of a
        // tile waits only for copies issued several tiles before; registers never wait on the
        // newest loads.
        constexpr int GPL = kST / 32;
        float* gring = reinterpret_cast<float*>(sm + Lay::kGRing);
        auto issue_gates = [&](int c) {
            float* dst = gring + (c % kGateTiles) * kST + GPL * ts;
            const int t0 = c < ntiles ? tile_t0(c) : 0, L = c < ntiles ? tile_len(c) : 0;
#pragma unroll
            for (int i = 0; i < GPL; ++i) {
                const bool in = GPL * ts + i < L;
                cp_async4(dst + i, in ? G + t0 + GPL * ts + i : G, in ? 4 : 0);
            }
            cp_async_commit();
        };
        if (GATED && ts < 32) {
#pragma unroll
            for (int f = 0; f < kGateTiles; ++f) issue_gates(f);
        }
        float kappa = 1.f, ldec_sum = 0.f;
        bool ok = true;
        for (int c = 0; c < ntiles && ok; ++c) {
            const int s = c % NS, L = tile_len(c);
            // tile decay (log2) and key weights
            float ldec;
            if (GATED) {
                if (ts < 32) {
                    cp_async_wait<kGateTiles - 1>();  // tile c's group (the oldest in flight) landed
                    const float* gs = gring + (c % kGateTiles) * kST + GPL * ts;
                    float y[GPL];
#pragma unroll
                    for (int i = 0; i < GPL; ++i) y[i] = gs[i] * kLog2e;
                    if constexpr (kST == 64) warp_cumsum64(y[0], y[1], lane, cum);
                    else warp_cumsum128(y, lane, cum);
                    issue_gates(c + kGateTiles);  // into the slot just read (each lane its own words)
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                ldec = cum[L - 1];
            } else {
                ldec = lg * (float)L;
            }
            const float dec = GATED ? exp2f(ldec) : pow_int_log2(lg, L);
            bool renorm;
            const float k_next = lazy_next_scale(kappa, dec, false, renorm);
            if (renorm && c > 0) {
                // T <- kappa dec T once the previous update has landed, so that with kappa = 1 the
                // next update adds onto the decayed state
                if (!wait_all(sbar(sUpd, (c - 1) % NS, NS), ((c - 1) / NS) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float sc = kappa * dec;
#pragma unroll 1
                for (int cb = 0; cb < DK / 32; ++cb) {
                    uint32_t w[32];
                    tmem_ld32(tmem + lane_off + cb * 32, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * sc);
                    tmem_st32(tmem + lane_off + cb * 32, w);
                }
                tmem_wait_st();
                tc_fence_before();
            }
            kappa = k_next;
            ldec_sum += ldec;
            if (ts < kST) {
                const float inv = 1.f / kappa;
                float z;
                if (GATED) z = REV ? exp2f(cum[ts]) : exp2f(cum[L - 1] - cum[ts]);
                else z = pow_int_log2(lg, REV ? ts + 1 : L - 1 - ts);
                zk[ts] = ts < L ? z * inv : 0.f;
            }
            if (!wait_all(sbar(sFull, s, NS), (c / NS) & 1)) {  // the V tile landed (and zk is complete)
                ok = false;
                break;
            }
            uint8_t* vt = sm + s * Lay::kStageBytes + Lay::kKBytes;
#pragma unroll
            for (int pass = 0; pass < kST / 64; ++pass) {
                // 16-byte chunks ci = e * 128 + ts of the two dv blocks (TT token rows of 128 bytes
                // each), so the token of a chunk is (ci mod 8 TT) / 8. All loads before any store.
                uint4 x[8];
                float z[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int ci = (pass * 8 + e) * 128 + ts;
                    z[e] = zk[(ci & (8 * kST - 1)) >> 3];
                    x[e] = *reinterpret_cast<const uint4*>(vt + ci * 16);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // bf16 pair products: the factor rounded to bf16, each product rounded once
                    const uint32_t z2 = pack_bf16(z[e], z[e]);
                    x[e].x = mul_bf16x2(x[e].x, z2);
                    x[e].y = mul_bf16x2(x[e].y, z2);
                    x[e].z = mul_bf16x2(x[e].z, z2);
                    x[e].w = mul_bf16x2(x[e].w, z2);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) *reinterpret_cast<uint4*>(vt + ((pass * 8 + e) * 128 + ts) * 16) = x[e];
            }
            fence_proxy_async();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ts == 0) mbar_arrive(bar(sbar(sZV, s, NS)));
        }
        if (GATED && ts < 32) asm volatile("cp.async.wait_all;" ::: "memory");  // no copy outlives the CTA
        // the end state S = kappa T, rows dk of column dv0 + d, and the total decay
        if (ok && wait_all(sbar(sUpd, (ntiles - 1) % NS, NS), ((ntiles - 1) / NS) & 1)) {
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < DK / 32; ++cb) {
                uint32_t w[32];
                tmem_ld32(tmem + lane_off + cb * 32, w);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) so[(size_t)(cb * 32 + i) * p.dv + d] = __uint_as_float(w[i]) * kappa;
            }
            if (slice == 0 && ts == 0) p.seg_ldec[(size_t)seg * gridDim.y + bh] = ldec_sum;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Lay::kTmemCols)
                     : "memory");
    }
}

}  // namespace tc
}  // namespace ret
