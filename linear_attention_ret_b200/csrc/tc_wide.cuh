// Tensor-core chunkwise retention with 128-token tiles, for a fixed decay gamma close
// to 1 (sm_100a). Included by tc_chunk.cuh, whose kernel runs this body for the CTAs
// of heads with log2(gamma) in [kWideMinLog2, 0] and dk in {128, 256}.
//
// Method: "RetNet retention mechanism" (aiqz.cc), section 块级循环 (chunkwise
// recurrence). Two changes against the 64-token body:
//
// 1. Tiles of 128 tokens. One tcgen05.mma takes about the same time for N = 64 and
//    N = 128 (on B200, 16 products of M64 N64 K16 take ~1160 cycles and of M128 N128
//    K16 ~1200), so Q K^T and the cross term cost half as much per token as with
//    64-token tiles.
//
// 2. One output accumulator, fed by zeta V in place of V. For a tile of L tokens let
//    zeta_m = gamma^(L-1-m) (the key weights of the state update) and hold the state as
//    S = kappa T (kappa a scalar, T in TMEM). With T the state before this tile's update,
//      O_j = (kappa / zeta_j) [ q_j T + sum_{m<=j} A_jm (zeta_m v_m / kappa) ],  A = Q K^T,
//    since gamma^(j-m) = zeta_m / zeta_j and gamma^(j+1) S_prev = gamma^L S_prev / zeta_j
//    = kappa T / zeta_j. So O_inter (from the bf16 copy of T) and O_intra (from the plain
//    causal mask of A and the same zeta V / kappa tile that the state update reads) add
//    into one TMEM region, and the drain scales token j by kappa / zeta_j. The state
//    epilogue turns the V tile into zeta V / kappa in place, so no V copy is kept.
//    With log2(gamma) >= kWideMinLog2 every factor stays within [2^-96, 2^96] (times
//    kappa in [2^-40, 1]), inside the normal range of bf16 and fp32.
//
// Products per tile (transposed so that M = 128 is the dv slice where it can be):
//   A   = Q K^T             M=128 (j) N=128 (m) K=dk   SS             -> TMEM region R
//   S^T += (zeta V / kappa)^T K   M=128 N=dk K=128     SS, both MN-major
//   Z^T  = T_op^T Q^T       M=128 N=128 K=dk           TS (bf16 T copy in TMEM) -> R
//   Z^T += (zeta V / kappa)^T P^T  M=128 N=128 K=128   SS, P = causal mask of A (bf16)
// TMEM: S^T (dk columns), its bf16 copy (dk/2), R (128 columns) -- 512 at dk = 256.
//
// REV (time-reversed direction, used for the gradients dK and dV): O_j = sum over later
// tokens i >= j of gamma^(i-j) (q_j . k_i) v_i. The tiles are visited from the last to
// the first and the state, referenced at the token before the current tile, is
// R = sum_{i >= t0} gamma^(i-t0+1) k_i^T v_i. Everything above holds with
// zeta_i = gamma^(i+1) (i the token's place in its tile) and the mask i >= j: the cross
// factor gamma^(L-1-j) R_next = kappa T / zeta_j with kappa T = gamma^L R_next.
// Shared memory: one Q and one K tile, each with its own full/empty barriers so that it
// reloads as soon as its last reader is done (K after the update, each dk half of Q after
// the cross term's steps over it); two V tiles (tile c in buffer c & 1, loaded right after K, so that V(c+1) lands
// and becomes zeta V / kappa while tile c's products still read ZV(c)); and one P tile
// that is also the staging tile of the O store (224 KB at dk = 256). zeta V / kappa is
// formed with bf16 pair products (the factor rounded to bf16, each product rounded once:
// the operand's rounding error grows from 2^-8 to about 2^-7, relative).
#pragma once

namespace ret {
namespace tc {

constexpr int kW = 128;                 // tokens per tile
constexpr int kBlk = kW * 128;          // one 128-row x 128-byte swizzled block (16 KB)
constexpr float kWideMinLog2 = -0.75f;  // gamma >= 2^-0.75 ~= 0.595

template <int DK>
struct WideLayout {
    static constexpr int kQ = 0;                        // Q tile: DK/64 blocks (rows = tokens)
    static constexpr int kK = kQ + DK / 64 * kBlk;      // K tile
    static constexpr int kV = kK + DK / 64 * kBlk;      // two V tiles, each then zeta V / kappa (2 blocks of 64 dv columns)
    static constexpr int kVBuf = 2 * kBlk;              // bytes of one V tile
    static constexpr int kP = kV + 2 * kVBuf;           // P (2 blocks of 64 m columns); O staging (4 x 64 x 64)
    static constexpr int kBar = kP + 2 * kBlk;
    static constexpr int kNumBars = 20;
    static constexpr int kAgTab = (kBar + kNumBars * 8 + 15) & ~15;  // attention group: drain row factors [128]
    static constexpr int kSgTab = kAgTab + kW * 4;      // state group: zeta / kappa [128]
    static constexpr int kBc = kSgTab + kW * 4;         // gated: the state group's tile decay, broadcast
    static constexpr int kTmemSlot = kBc + 16;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kSmemAlloc = kBytes + 1024;    // slack to align the base to 1024 B
    static constexpr int kColS = 0;
    static constexpr int kColSop = DK;
    static constexpr int kColR = DK + DK / 2;
    static constexpr int kTmemCols = kColR + kW <= 256 ? 256 : 512;
    static_assert(kColR + kW <= 512, "TMEM overflow");
    static_assert(kAgTab % 16 == 0 && kSgTab % 16 == 0, "row-factor tables are read as float4");
    static_assert(kSmemAlloc <= 227 * 1024, "shared memory overflow");
};

enum WideBar {
    wQFull = 0, wKFull, wQEmpty, wKEmpty,      // wQFull, wQEmpty: the low dk half of Q (wQFullHi, wQEmptyHi: the high)
    wVFull0, wVFull1, wVEmpty0, wVEmpty1,      // per V buffer (tile c uses buffer c & 1)
    wAFull, wARead, wPReady, wOFull, wOFree,
    wSFull, wSReady, wZV0, wZV1, wDrain,
    wQFullHi, wQEmptyHi
};

// Lazy decay normalisation (S = kappa T). Given the current kappa and the next tile's
// decay gamma^L, returns the next kappa: kappa gamma^L, or 1 when that would fall below
// 2^-40 (then T itself is rescaled by kappa gamma^L). Both epilogue groups evaluate it,
// with the same operations, so they agree on kappa bit for bit.
__device__ __forceinline__ float lazy_next_scale(float kappa, float decay, bool force, bool& renorm) {
    renorm = force || !(kappa * decay >= 9.094947e-13f);  // 2^-40
    return renorm ? 1.f : kappa * decay;
}

// Gated: raw gates 4l .. 4l+3 (natural-log units) of the 128-token tile starting at t0, for
// lane l of one warp; zero at and past the segment end tend.
__device__ __forceinline__ void load_gates4(const float* G, int t0, int tend, int lane, float (&g)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 4 * lane + i;
        g[i] = t < tend ? G[t] : 0.f;
    }
}

// Gated: in-tile inclusive cumulative log2-decay c of a 128-token tile by one warp, from the
// raw gates load_gates4 gave lane l; lane l gets c at tokens 4l .. 4l+3. Returns the tile's
// total, c after token 127 (equal to c after the last valid token: gates past it are zero).
__device__ __forceinline__ float tile_scan128(const float (&g)[4], float (&c)[4], int lane) {
    const float y0 = g[0] * kLog2e, y1 = g[1] * kLog2e, y2 = g[2] * kLog2e, y3 = g[3] * kLog2e;
    const float p1 = y0 + y1, p2 = p1 + y2, p3 = p2 + y3;
    float incl = p3;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const float excl = incl - p3;
    c[0] = excl + y0;
    c[1] = excl + p1;
    c[2] = excl + p2;
    c[3] = excl + p3;
    return __shfl_sync(0xffffffffu, c[3], 31);
}

template <int DK, bool REV, bool GATED = false>
__device__ __forceinline__ void wide_body(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                          const CUtensorMap& tm_o, const Params& p, float lg) {
    using Lay = WideLayout<DK>;
    // dk = 256: Q in two dk halves with their own barriers (each reloads once the cross term
    // has read it); at dk = 128 one Q barrier measured faster
    constexpr bool kQHalves = DK == 256;
    constexpr int kQLo = kQHalves ? DK / 128 : DK / 64;  // dk blocks of the low part (all of Q without halves)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int b) { return sbase + Lay::kBar + 8 * b; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::kTmemSlot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // seg: place of this segment in the order the segments are chained (its start state is
    // the chain's seg-th); tseg: its place in time (REV chains them from the last back)
    const int slice = blockIdx.x, bh = blockIdx.y, seg = blockIdx.z;
    const int tseg = REV ? p.units - 1 - seg : seg;
    const int dv0 = slice * kDvS;
    const int tbeg = tseg * p.seg_chunks * kC;                // first token of this segment
    const int tend = min(tbeg + p.seg_chunks * kC, p.N);      // one past its last token
    const int ntiles = (tend - tbeg + kW - 1) / kW;
    const bool last_seg = seg == p.units - 1;                 // the chain's last: writes state_out
    // token start of the c-th tile visited (REV: from the last tile of the segment back)
    auto tile_t0 = [&](int c) { return tbeg + (REV ? ntiles - 1 - c : c) * kW; };
    auto tile_len = [&](int c) { return min(kW, tend - tile_t0(c)); };
    // gated: this head's gates g [N] (log-decay per token); the tile factors below replace
    // gamma^L by the tile decay exp2(c_last) and gamma^(L-1-m) by zeta_m = exp2(c_last - c_m),
    // with c the tile's inclusive cumulative log2-decay (REV: gamma^(i+1) by zeta_i = exp2(c_i))
    const float* G = GATED ? p.decay_in + (size_t)bh * p.N : nullptr;

    if (threadIdx.x == 0) {
        for (int b = 0; b < Lay::kNumBars; ++b) mbar_init(bar(b), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_o)) : "memory");
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
            // 64 x 64 boxes; two of them (tokens t0 and t0 + 64) fill one 128-row block.
            // Rows past the segment end are loaded too and masked by the epilogues; rows
            // past N read as zero.
            int issued[4] = {-1, -1, -1, -1};  // K, Q low half, V, Q high half: last tile whose copies were issued
            for (int c = 0; c < ntiles; ++c) {
                const int t0 = tile_t0(c);
                const uint32_t ph = (c - 1) & 1;
                if (c > 0 && !mbar_wait(bar(wKEmpty), ph, abort_flag)) break;
                mbar_expect_tx(bar(wKFull), DK / 64 * kBlk);
#pragma unroll
                for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load_3d(sbase + Lay::kK + kb * kBlk + h * kTile64, &tm_k, kb * 64, t0 + 64 * h, bh, bar(wKFull));
                issued[0] = c;
                // V tile c into buffer c & 1 (free once O_intra(c - 2) has read it), before Q: the
                // state epilogue turns it into zeta V / kappa while tile c - 1 is still running
                {
                    const int vb = c & 1;
                    if (c > 1 && !mbar_wait(bar(wVEmpty0 + vb), ((c >> 1) - 1) & 1, abort_flag)) break;
                    mbar_expect_tx(bar(wVFull0 + vb), Lay::kVBuf);
#pragma unroll
                    for (int db = 0; db < 2; ++db)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tma_load_3d(sbase + Lay::kV + vb * Lay::kVBuf + db * kBlk + h * kTile64, &tm_v, dv0 + 64 * db,
                                        t0 + 64 * h, bh, bar(wVFull0 + vb));
                }
                issued[2] = c;
                // Q: the low part (all of Q without halves), then the high half
                if (c > 0 && !mbar_wait(bar(wQEmpty), ph, abort_flag)) break;
                mbar_expect_tx(bar(wQFull), kQLo * kBlk);
#pragma unroll
                for (int kb = 0; kb < kQLo; ++kb)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load_3d(sbase + Lay::kQ + kb * kBlk + h * kTile64, &tm_q, kb * 64, t0 + 64 * h, bh, bar(wQFull));
                issued[1] = c;
                if constexpr (kQHalves) {
                    if (c > 0 && !mbar_wait(bar(wQEmptyHi), ph, abort_flag)) break;
                    mbar_expect_tx(bar(wQFullHi), (DK / 64 - kQLo) * kBlk);
#pragma unroll
                    for (int kb = kQLo; kb < DK / 64; ++kb)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tma_load_3d(sbase + Lay::kQ + kb * kBlk + h * kTile64, &tm_q, kb * 64, t0 + 64 * h, bh,
                                        bar(wQFullHi));
                    issued[3] = c;
                }
            }
            if (*abort_flag) {
                // drain the copies in flight before the CTA may exit
                if (issued[0] >= 0) mbar_drain(bar(wKFull), issued[0] & 1);
                if (issued[1] >= 0) mbar_drain(bar(wQFull), issued[1] & 1);
                if (kQHalves && issued[3] >= 0) mbar_drain(bar(wQFullHi), issued[3] & 1);
                for (int c = std::max(issued[2] - 1, 0); c <= issued[2]; ++c) mbar_drain(bar(wVFull0 + (c & 1)), (c >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc(128, kW, 0, 0);
            constexpr uint32_t id_oi = idesc(128, kW, 0, 0);
            constexpr uint32_t id_ov = idesc(128, kW, 1, 0);
            constexpr uint32_t id_up = idesc(128, DK, 1, 1);
            const uint32_t tS = tmem + Lay::kColS, tSop = tmem + Lay::kColSop, tR = tmem + Lay::kColR;
            const uint32_t sQ = sbase + Lay::kQ, sK = sbase + Lay::kK, sP = sbase + Lay::kP;
            for (int c = 0; c < ntiles; ++c) {
                const uint32_t ph = c & 1;
                // A = Q K^T (both K-major; 16-element K steps, 64-column blocks 16 KB apart);
                // region R is free once the previous tile's output has been read out.
                if (!mbar_wait(bar(wQFull), ph, abort_flag) || !mbar_wait(bar(wKFull), ph, abort_flag)) break;
                if (c > 0 && !mbar_wait(bar(wOFree), (c - 1) & 1, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4 * kQLo; ++ks) {  // the low part of Q
                    const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
                    mma_ss(tR, sdesc(sQ + off, 16, 1024), sdesc(sK + off, 16, 1024), id_qk, ks > 0);
                }
                if constexpr (kQHalves) {
                    if (!mbar_wait(bar(wQFullHi), ph, abort_flag)) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 4 * kQLo; ks < DK / 16; ++ks) {  // the high half
                        const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
                        mma_ss(tR, sdesc(sQ + off, 16, 1024), sdesc(sK + off, 16, 1024), id_qk, 1);
                    }
                }
                mma_commit(bar(wAFull));
                // S^T += (zeta V / kappa)^T K while the epilogue reads A: A operand = the
                // scaled V tile MN-major (dv blocks 16 KB apart), B = K tile MN-major.
                const int vb = c & 1;
                const uint32_t sZ = sbase + Lay::kV + vb * Lay::kVBuf;  // this tile's zeta V / kappa
                if (!mbar_wait(bar(wZV0 + vb), (c >> 1) & 1, abort_flag) || !mbar_wait(bar(wSReady), ph, abort_flag))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kW / 16; ++ks)
                    mma_ss(tS, sdesc(sZ + ks * 2048, kBlk, 1024), sdesc(sK + ks * 2048, kBlk, 1024), id_up, 1);
                mma_commit(bar(wKEmpty));
                // Z^T = T_op^T Q^T into R once A has been read (A from TMEM, B = Q tile K-major)
                if (!mbar_wait(bar(wARead), ph, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4 * kQLo; ++ks) {
                    const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
                    mma_ts(tR, tSop + ks * 8, sdesc(sQ + off, 16, 1024), id_oi, ks > 0);
                }
                mma_commit(bar(wQEmpty));  // the low part of Q may reload
#pragma unroll
                for (int ks = 4 * kQLo; ks < DK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
                    mma_ts(tR, tSop + ks * 8, sdesc(sQ + off, 16, 1024), id_oi, 1);
                }
                // the update and the cross term are done: the state epilogue may read S and
                // overwrite its bf16 copy; the high half of Q may reload
                mma_commit(bar(wSFull));
                if constexpr (kQHalves) mma_commit(bar(wQEmptyHi));
                // Z^T += (zeta V / kappa)^T P^T (B = P K-major, m blocks 16 KB apart)
                if (!mbar_wait(bar(wPReady), ph, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kW / 16; ++ks)
                    mma_ss(tR, sdesc(sZ + ks * 2048, kBlk, 1024), sdesc(sP + (ks >> 2) * kBlk + (ks & 3) * 32, 16, 1024),
                           id_ov, 1);
                mma_commit(bar(wOFull));
                mma_commit(bar(wVEmpty0 + vb));
            }
            // every issued MMA must complete before TMEM can be released
            mma_commit(bar(wDrain));
            mbar_drain(bar(wDrain), 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ attention epilogue (warps 2..5)
        const int te = threadIdx.x - 64;   // 0..127
        const int quarter = warp & 3;      // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;  // TMEM lane: token row j of A, dv column d of Z^T
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tR = tmem + lane_off + Lay::kColR;
        float* rowf = reinterpret_cast<float*>(sm + Lay::kAgTab);
        auto wait_all = [&](int b, uint32_t parity) {  // every thread reaches the barrier; uniform result
            mbar_wait(bar(b), parity, abort_flag);
            group_sync(1);
            return *abort_flag == 0;
        };
        float kappa = 1.f;
        // gated: the group's first warp scans each tile's gates (prefetched one tile ahead, raw)
        // and alone holds kappa; the other threads only read the row factors it writes
        float gnext[4] = {0.f, 0.f, 0.f, 0.f};
        if (GATED && te < 32) load_gates4(G, tile_t0(0), tend, lane, gnext);
        for (int c = 0; c < ntiles; ++c) {
            const int t0 = tile_t0(c), L = tile_len(c);
            float gc[4] = {0.f, 0.f, 0.f, 0.f}, gl = 0.f;
            if constexpr (GATED) {
                if (te < 32) {
                    gl = tile_scan128(gnext, gc, lane);
                    if (c + 1 < ntiles) load_gates4(G, tile_t0(c + 1), tend, lane, gnext);
                    if (c > 0) {
                        bool rn;
                        kappa = lazy_next_scale(kappa, exp2f(gl), false, rn);
                    }
                }
            } else if (c > 0) {
                bool rn;
                kappa = lazy_next_scale(kappa, pow_int_log2(lg, L), false, rn);
            }
            // ---------------- P = causal mask of A in bf16, row j = r (K-major, 128-byte swizzle);
            // REV keeps the upper triangle m >= j instead
            if (!wait_all(wAFull, c & 1)) break;
            tc_fence_after();
            uint32_t pk[64];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t a0[32], a1[32];
                tmem_ld32(tR + hh * 64, a0);
                tmem_ld32(tR + hh * 64 + 32, a1);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int m = hh * 64 + 2 * u;
                    auto keep = [&](int mm) { return REV ? mm >= r : mm <= r; };
                    pk[hh * 32 + u] = pack_bf16(keep(m) ? __uint_as_float(a0[2 * u]) : 0.f,
                                                keep(m + 1) ? __uint_as_float(a0[2 * u + 1]) : 0.f);
                    pk[hh * 32 + 16 + u] = pack_bf16(keep(m + 32) ? __uint_as_float(a1[2 * u]) : 0.f,
                                                     keep(m + 33) ? __uint_as_float(a1[2 * u + 1]) : 0.f);
                }
            }
            // A is in registers: the cross term may overwrite R. The previous tile's O store
            // must have read the staging tile (the P region) before P is written.
            tc_fence_before();
            if (te == 0) tma_store_wait_read();
            group_sync(1);
            if (te == 0) mbar_arrive(bar(wARead));
            {
                uint8_t* prow = sm + Lay::kP + r * 128;
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    *reinterpret_cast<uint4*>(prow + (q >> 3) * kBlk + (((q & 7) ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            fence_proxy_async();
            group_sync(1);
            if (te == 0) mbar_arrive(bar(wPReady));
            // ---------------- O_j = (kappa / zeta_j) Z_j -> bf16 -> staging -> TMA store
            if constexpr (GATED) {
                if (te < 32) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int tok = 4 * lane + i;
                        // kappa / zeta_j: zeta_j = exp2(c_last - c_j), REV exp2(c_j)
                        rowf[tok] = tok < L ? kappa * exp2f(REV ? -gc[i] : gc[i] - gl) : 0.f;
                    }
                }
            } else {
                rowf[te] = te < L ? kappa * pow_int_log2(-lg, REV ? te + 1 : L - 1 - te) : 0.f;
            }
            if (!wait_all(wOFull, c & 1)) break;
            tc_fence_after();
            {
                // Z^T (dv lanes x 128 token columns) read as 16-lane x 8-column fragments:
                // z[hf][th] holds lanes quarter*32 + 16 hf + {g, g + 8} (g = lane / 4) and token
                // columns 64 th + 8k + 2 (lane % 4) + {0, 1}, k = 0..7 -- pairs of adjacent tokens
                // of one dv column, the register layout stmatrix .trans writes as 8 x 8 blocks of
                // (token rows x dv columns) into the staging tiles.
                uint32_t z[2][2][32];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int th = 0; th < 2; ++th) tmem_ld16x256b_x8(tR + ((uint32_t)(16 * hf) << 16) + 64 * th, z[hf][th]);
                tmem_wait_ld();
                tc_fence_before();
                group_sync(1);
                if (te == 0) mbar_arrive(bar(wOFree));
                const int i2 = 2 * (lane & 3);
#pragma unroll
                for (int th = 0; th < 2; ++th) {
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        // row factors of tokens 64 th + 8k' + i2 + {0, 1}, k' = k, k + 1
                        const float2 f0 = reinterpret_cast<const float2*>(rowf)[(64 * th + 8 * k + i2) >> 1];
                        const float2 f1 = reinterpret_cast<const float2*>(rowf)[(64 * th + 8 * k + 8 + i2) >> 1];
                        // block b = 2 (k' - k) + (dv half of the 16 lanes); thread lane supplies the
                        // address of block lane / 8, row lane % 8 (token 64 th + 8 (k + b / 2) + lane % 8)
                        const int b = lane >> 3, q = lane & 7;
                        const int jr = 8 * (k + (b >> 1)) + q;  // token row inside the 64-token box
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const uint32_t* zz = z[hf][th];
                            const uint32_t r0 = pack_bf16(f0.x * __uint_as_float(zz[4 * k]), f0.y * __uint_as_float(zz[4 * k + 1]));
                            const uint32_t r1 = pack_bf16(f0.x * __uint_as_float(zz[4 * k + 2]), f0.y * __uint_as_float(zz[4 * k + 3]));
                            const uint32_t r2 = pack_bf16(f1.x * __uint_as_float(zz[4 * k + 4]), f1.y * __uint_as_float(zz[4 * k + 5]));
                            const uint32_t r3 = pack_bf16(f1.x * __uint_as_float(zz[4 * k + 6]), f1.y * __uint_as_float(zz[4 * k + 7]));
                            const int dvb = quarter * 32 + 16 * hf + 8 * (b & 1);  // first dv column of the block
                            const uint32_t box = sbase + Lay::kP + (2 * th + (dvb >> 6)) * kTile64;
                            stmatrix_x4_trans(box + jr * 128 + (((((dvb & 63) >> 3) ^ (jr & 7))) << 4), r0, r1, r2, r3);
                        }
                    }
                }
            }
            fence_proxy_async();
            group_sync(1);
            if (te == 0) {
                // tokens past the segment end belong to the next segment: store only the
                // 64-token halves that start inside this tile (rows past N are clipped)
#pragma unroll
                for (int th = 0; th < 2; ++th) {
                    if (th * 64 >= L) break;
                    tma_out_3d(p.o_add, &tm_o, dv0, t0 + 64 * th, bh, sbase + Lay::kP + (2 * th) * kTile64);
                    tma_out_3d(p.o_add, &tm_o, dv0 + 64, t0 + 64 * th, bh, sbase + Lay::kP + (2 * th + 1) * kTile64);
                }
                tma_store_commit();
            }
        }
        if (te == 0) tma_store_wait_all();
    } else {
        // ------------------------------------------------------------ state epilogue (warps 6..9)
        const int ts = threadIdx.x - 192;  // 0..127
        const int quarter = warp & 3;
        const int d = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float* zk = reinterpret_cast<float*>(sm + Lay::kSgTab);  // zeta_m / kappa
        float* bc = reinterpret_cast<float*>(sm + Lay::kBc);     // gated: the next tile's decay
        // gated: the group's first warp scans the next tile's gates (prefetched one tile ahead)
        float graw[4] = {0.f, 0.f, 0.f, 0.f}, sgc[4] = {0.f, 0.f, 0.f, 0.f}, sgl = 0.f;
        auto wait_all = [&](int b, uint32_t parity) {
            mbar_wait(bar(b), parity, abort_flag);
            group_sync(2);
            return *abort_flag == 0;
        };
        // The V tile of tile c becomes zeta V / kappa in place: 16-byte chunks ci = e * 128 + ts,
        // two 16 KB blocks of 128 token rows, so the token of a chunk is (ci mod 1024) / 8.
        auto build_zv = [&](int c, float kappa) {
            const int L = tile_len(c);
            if constexpr (GATED) {
                if (ts < 32) {  // sgc, sgl: the scan of tile c
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int tok = 4 * lane + i;
                        zk[tok] = tok < L ? exp2f(REV ? sgc[i] : sgl - sgc[i]) * (1.f / kappa) : 0.f;
                    }
                }
            } else {
                zk[ts] = ts < L ? pow_int_log2(lg, REV ? ts + 1 : L - 1 - ts) * (1.f / kappa) : 0.f;
            }
            if (!wait_all(wVFull0 + (c & 1), (c >> 1) & 1)) return false;
            uint8_t* vt = sm + Lay::kV + (c & 1) * Lay::kVBuf;
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                uint4 x[8];
                float z[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {  // all loads before any store (aliasing)
                    const int ci = (pass * 8 + e) * kEpiThreads + ts;
                    z[e] = zk[(ci & 1023) >> 3];
                    x[e] = *reinterpret_cast<const uint4*>(vt + ci * 16);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // bf16 pair products (the factor rounded to bf16, the product rounded once)
                    const uint32_t z2 = pack_bf16(z[e], z[e]);
                    x[e].x = mul_bf16x2(x[e].x, z2);
                    x[e].y = mul_bf16x2(x[e].y, z2);
                    x[e].z = mul_bf16x2(x[e].z, z2);
                    x[e].w = mul_bf16x2(x[e].w, z2);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    *reinterpret_cast<uint4*>(vt + ((pass * 8 + e) * kEpiThreads + ts) * 16) = x[e];
            }
            fence_proxy_async();
            group_sync(2);
            if (ts == 0) mbar_arrive(bar(wZV0 + (c & 1)));
            return true;
        };

        // Initial state: kappa = 1, T = gamma^L0 S_in, bf16 copy = bf16(T), S_in from
        // segment_start_state().
        float kappa;
        {
            bool rn;
            float dec0;
            if constexpr (GATED) {
                if (ts < 32) {
                    load_gates4(G, tile_t0(0), tend, lane, graw);
                    sgl = tile_scan128(graw, sgc, lane);
                    if (lane == 0) bc[0] = exp2f(sgl);
                    if (ntiles > 1) load_gates4(G, tile_t0(1), tend, lane, graw);
                }
                group_sync(2);
                dec0 = bc[0];
            } else {
                dec0 = pow_int_log2(lg, tile_len(0));
            }
            kappa = lazy_next_scale(1.f, dec0, true, rn);
            const float* sin = segment_start_state(p, seg, bh, DK, dv0 + d);
#pragma unroll 1
            for (int cb = 0; cb < DK / 32; ++cb) {
                uint32_t w[32], h[16];
#pragma unroll
                for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(sin ? sin[(size_t)(cb * 32 + c) * p.dv] : 0.f);
#pragma unroll
                for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(__uint_as_float(w[c]) * dec0);
#pragma unroll
                for (int c = 0; c < 16; ++c) h[c] = pack_bf16(__uint_as_float(w[2 * c]), __uint_as_float(w[2 * c + 1]));
                tmem_st32(tmem + lane_off + Lay::kColS + cb * 32, w);
                tmem_st16(tmem + lane_off + Lay::kColSop + cb * 16, h);
            }
            tmem_wait_st();
            tc_fence_before();
            group_sync(2);
            if (ts == 0) mbar_arrive(bar(wSReady));
        }
        bool ok = build_zv(0, kappa);
        for (int c = 0; c < ntiles && ok; ++c) {
            const bool last = c == ntiles - 1;
            bool rn = false;
            float dec_next = 0.f, k_next = 1.f;
            if (!last) {
                if constexpr (GATED) {
                    if (ts < 32) {  // scan tile c + 1; its decay reaches the group at the barrier below
                        sgl = tile_scan128(graw, sgc, lane);
                        if (c + 2 < ntiles) load_gates4(G, tile_t0(c + 2), tend, lane, graw);
                        if (lane == 0) bc[0] = exp2f(sgl);
                    }
                } else {
                    dec_next = pow_int_log2(lg, tile_len(c + 1));
                    k_next = lazy_next_scale(kappa, dec_next, false, rn);
                }
            }
            if (!wait_all(wSFull, c & 1)) break;
            if (GATED && !last) {
                dec_next = bc[0];
                k_next = lazy_next_scale(kappa, dec_next, false, rn);
            }
            tc_fence_after();
            if (last) {
                float* so = last_seg ? p.state_out : nullptr;
                if (so) {
                    so += ((size_t)bh * DK) * p.dv + dv0 + d;
#pragma unroll 1
                    for (int cb = 0; cb < DK / 32; ++cb) {
                        uint32_t w[32];
                        tmem_ld32(tmem + lane_off + Lay::kColS + cb * 32, w);
                        tmem_wait_ld();
#pragma unroll
                        for (int cc = 0; cc < 32; ++cc) so[(size_t)(cb * 32 + cc) * p.dv] = __uint_as_float(w[cc]) * kappa;
                    }
                }
                break;
            }
            // Next bf16 copy = bf16(T'), T' = T, or kappa gamma^L T when kappa renormalises
            // (then T' is also written back).
            const float tscale = kappa * dec_next;
#pragma unroll 1
            for (int cb = 0; cb < DK / 64; ++cb) {
                uint32_t w0[32], w1[32], h[16];
                tmem_ld32(tmem + lane_off + Lay::kColS + cb * 64, w0);
                tmem_ld32(tmem + lane_off + Lay::kColS + cb * 64 + 32, w1);
                tmem_wait_ld();
                if (rn) {
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) {
                        w0[cc] = __float_as_uint(__uint_as_float(w0[cc]) * tscale);
                        w1[cc] = __float_as_uint(__uint_as_float(w1[cc]) * tscale);
                    }
                    tmem_st32(tmem + lane_off + Lay::kColS + cb * 64, w0);
                    tmem_st32(tmem + lane_off + Lay::kColS + cb * 64 + 32, w1);
                }
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) h[cc] = pack_bf16(__uint_as_float(w0[2 * cc]), __uint_as_float(w0[2 * cc + 1]));
                tmem_st16(tmem + lane_off + Lay::kColSop + cb * 32, h);
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) h[cc] = pack_bf16(__uint_as_float(w1[2 * cc]), __uint_as_float(w1[2 * cc + 1]));
                tmem_st16(tmem + lane_off + Lay::kColSop + cb * 32 + 16, h);
            }
            tmem_wait_st();
            tc_fence_before();
            group_sync(2);
            if (ts == 0) mbar_arrive(bar(wSReady));
            kappa = k_next;
            ok = build_zv(c + 1, kappa);
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
