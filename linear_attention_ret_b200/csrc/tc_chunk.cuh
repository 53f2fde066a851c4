// Tensor-core (tcgen05 + TMA + TMEM) chunkwise retention for sm_100a.
//
// Method: "RetNet retention mechanism" (aiqz.cc), section 块级循环 (chunkwise
// recurrence), and the gated chunk_gate_retention (pwwt.cn page). For chunk i
// (64 tokens, local rows j, m), with decays as in the CUDA-core kernel:
//   O_[i] = (Q K^T (.) D) V + diag(r) Q S_[i-1]
//   S_[i] = decay S_[i-1] + K^T diag(zeta) V
//
// Work split. One CTA owns one head and a 128-column slice of dv and walks the
// chunks of its sequence range in order. The products run transposed so that
// the large ones have M = 128 (one TMEM lane per dv column of the slice):
//   A        = Q K^T                 M=64  N=64  K=dk  (SS)   -> TMEM, masked by the epilogue into P (bf16, smem)
//   O_inter^T = S_op^T Q^T           M=128 N=64  K=dk  (TS: S_op = bf16 copy of the state, in TMEM)
//   O_intra^T = V^T P^T              M=128 N=64  K=64  (SS, V read MN-major straight from the TMA tile)
//   S^T      += (zeta V)^T K         M=128 N=dk  K=64  (SS, K read MN-major from the same TMA tile)
// The fp32 state lives in TMEM for the whole sequence as S = c T (c a scalar
// kept in registers): each chunk the epilogue reads T once and writes the
// bf16 copy of S (the next cross term's MMA operand); the update adds
// (zeta V / c) onto T, and T is rescaled in place only when c would underflow.
// The decay mask is generated in registers. For a fixed gamma in [1/2, 1] the two
// output products add into one accumulator (decay factors moved onto the state copy,
// P and the drain; derivation at the kernel), which frees TMEM to double-buffer the
// attention products even at dk = 256.
//
// Roles (320 threads): warp 0 issues TMA loads (two stages of Q, K, V tiles);
// warp 1 allocates TMEM and issues every tcgen05.mma from one thread; warps 2-5
// are the attention epilogue (mask P from Q K^T, combine and store O); warps
// 6-9 are the state epilogue (zeta-scaled V into a double buffer, and the TMEM
// round trip of the state). The two epilogue groups run concurrently; each
// warp reads the TMEM lane quarter (warp index % 4). All waits are bounded: on
// timeout the kernel sets the device error word, the roles stop, in-flight
// copies and MMAs are drained (bounded again) and TMEM is released.
#pragma once

#include <algorithm>
#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>

#include <utility>

#include "common.cuh"

namespace ret {
namespace tc {

constexpr int kC = 64;          // chunk rows per tile
constexpr int kDvS = 128;       // dv columns per CTA (TMEM lanes)
constexpr int kThreads = 320;
constexpr int kEpiThreads = 128;  // threads per epilogue group
constexpr int kTile64 = kC * 128;  // one 64-row x 128-byte swizzled tile (8 KB)
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait

template <int DK>
struct Layout {
    static constexpr int kQBytes = DK / 64 * kTile64;
    static constexpr int kKBytes = DK / 64 * kTile64;
    static constexpr int kVBytes = 2 * kTile64;
    static constexpr int kStageBytes = kQBytes + kKBytes + kVBytes;
    static constexpr int kStage0 = 0;
    // Attention buffers. Two of them let chunk i+1's Q K^T and mask overlap chunk i's output
    // products and drain. A buffer holds Q K^T, then O_inter^T in the same columns, plus a
    // separate O_intra^T region (128 columns) -- or, with the merged output accumulator
    // (fixed gamma, see the kernel), one region of 64 columns that both products add into.
    // With dk <= 128 TMEM has room for two split buffers; with dk = 256 the state takes 384
    // columns and the remaining 128 hold two merged buffers or one split buffer.
    static constexpr int kPTiles = 2;
    // TMA stages of Q, K, V tiles: three where shared memory allows, so that loads run two
    // chunks ahead of the products that read them.
    static constexpr int kStages = DK <= 128 ? 3 : 2;
    static constexpr int kP = kStages * kStageBytes;        // P tiles (64 x 64 bf16, SW128 K-major), one per buffer
    static constexpr int kZV = kP + kPTiles * kTile64;      // zeta-scaled V, two buffers (V tile layout)
    static constexpr int kOst = kZV + 2 * kVBytes;          // O staging for the TMA store (128-byte swizzle)
    static constexpr int kBar = kOst + kVBytes;             // mbarriers
    static constexpr int kNumBars = 22;
    static constexpr int kAgTab = kBar + kNumBars * 8;      // attention group: cum[2][64] | r[2][64] | pw[68]
    static constexpr int kSgTab = kAgTab + 324 * 4;         // state group: cum[64] | zeta[64] | decay
    static constexpr int kTmemSlot = kSgTab + 132 * 4;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static constexpr int kSmemAlloc = kBytes + 1024;        // slack to align the base to 1024 B
    // TMEM columns
    static constexpr int kColS = 0;                 // fp32 state S^T: DK columns
    static constexpr int kColSop = DK;              // bf16 state copy: DK/2 columns
    static constexpr int kColA = DK + DK / 2;       // attention buffers from here (Q K^T, O_inter^T, O_intra^T)
    static constexpr int kColsUsed = kColA + (DK <= 128 ? 4 : 2) * kC;
    static constexpr int kTmemCols = kColsUsed <= 256 ? 256 : 512;
    static_assert(kColsUsed <= 512, "TMEM overflow");
    static_assert(kSmemAlloc <= 227 * 1024, "shared memory overflow");
};

enum Bar {
    kFull0 = 0, kFull1, kFull2, kEmpty0, kEmpty1, kEmpty2,  // TMA stages
    kAFull0, kAFull1, kARead0, kARead1,          // attention epilogue <-> MMA, per attention buffer
    kPReady0, kPReady1, kOFull0, kOFull1, kOFree0, kOFree1,
    kSFull, kSReady, kZV0, kZV1,                 // state epilogue <-> MMA
    kDrain
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait. Returns false (and sets the abort flag and the device error
// word on the first timeout) if the phase did not complete within limit_ns or
// another role already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            raise_error(kErrWaitTimeout);
            return false;
        }
    }
}

// Wait used while draining after an abort: bounded, never raises.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kWaitNs) {
    }
}

// Named barrier of one epilogue group (id 1: attention group, id 2: state group).
__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, int x, int y, int z, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(src)
                 : "memory");
}
// Adds the tile into global memory instead of storing it (the addition is done in L2,
// element by element in the tensor's type, rounded once).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, int x, int y, int z, uint32_t src) {
    asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3}], [%4];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(src)
                 : "memory");
}
// The output tile copy: a store, or an addition onto what the output already holds.
__device__ __forceinline__ void tma_out_3d(bool add, const CUtensorMap* map, int x, int y, int z, uint32_t src) {
    if (add)
        tma_reduce_add_3d(map, x, y, z, src);
    else
        tma_store_3d(map, x, y, z, src);
}
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}


// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start address,
// leading and stride byte offsets in 16-byte units, version 1 at bit 46, layout 2 at bit 61).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D; majors 0 = K, 1 = MN.
__host__ __device__ constexpr uint32_t idesc(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(id), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM words: thread t of the warp gets lane (base+t), columns c..c+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// 16 lanes x 2 halves: thread t gets lane (base + t % 16), columns c + 32 * (t / 16) .. +31.
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// 16 lanes x 8 columns, repeated 8 times along the columns (64 columns): with g = t / 4 and
// i = t % 4, thread t gets r[4k] = (lane g, column 8k + 2i), r[4k+1] = (lane g, column 8k + 2i + 1),
// r[4k+2] = (lane g + 8, column 8k + 2i), r[4k+3] = (lane g + 8, column 8k + 2i + 1).
__device__ __forceinline__ void tmem_ld16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Four 8 x 8 blocks of 16-bit values to shared memory, transposed: block b's row q (16 bytes)
// goes to the address thread 8b + q supplies; thread t's register for block b holds that
// block's elements (row 2 (t % 4), column t / 4) in its low half and (row 2 (t % 4) + 1,
// column t / 4) in its high half.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};"
                 ::"r"(addr), "r"(r0), "r"(r1), "r"(r2), "r"(r3) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Two bf16 products in one instruction (each rounded to bf16 once).
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
}

// ------------------------------------------------------------------ kernel

struct Params {
    const float* decay_in;   // gamma [H] or g [B, H, N]
    const float* state_in;   // [B, H, dk, dv] or null
    float* state_out;        // [B, H, dk, dv] or null
    float* seg_state;        // [G-1, B*H, dk, dv]: local end state of segments 0..G-2 (scratch)
    float* seg_ldec;         // [G-1, B*H]: log2 of each of those segments' total decay (scratch)
    int H, N, dv;
    int seg_chunks;          // chunks per sequence segment (blockIdx.z = segment)
    int sub_per_seg;         // state-only sub-segments per full-pass segment (their start states are in seg_state)
    int units;               // segments the sequence is cut into at seg_chunks each (REV counts them from the end)
    int o_add;               // nonzero: output tiles are added onto o (which the caller has initialised)
};

// In-chunk inclusive cumulative sum of the gate in log2 units, by one warp:
// lane l holds g[2l], g[2l+1] (already scaled by log2(e)); writes cum[0..63].
__device__ __forceinline__ void warp_cumsum64(float g0, float g1, int lane, float* cum) {
    const float pair = g0 + g1;
    float incl = pair;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    cum[2 * lane] = incl - pair + g0;
    cum[2 * lane + 1] = incl;
}

}  // namespace tc
}  // namespace ret

#include "tc_wide.cuh"
#include "tc_state.cuh"

namespace ret {
namespace tc {

// Start state of segment seg of a split sequence, column `col` of head bh: state_in (or
// none: zero) for the first segment; for segment g > 0 the prefix pass has left it in
// seg_state[g F - 1] (F = sub_per_seg: the state-only pass may cut segments finer). Rows
// are dv apart.
__device__ __forceinline__ const float* segment_start_state(const Params& p, int seg, int bh, int dk, int col) {
    if (seg > 0) return p.seg_state + ((size_t)(seg * p.sub_per_seg - 1) * gridDim.y + bh) * dk * p.dv + col;
    return p.state_in ? p.state_in + ((size_t)bh * dk) * p.dv + col : nullptr;
}

// Whether an instantiation may run the 128-token body: dk of 128 or 256, not the state-only pass.
constexpr bool wide_capable(int dk, bool gated, bool state_only) {
    return !state_only && dk >= 128;
}

// Gated: whether every gate of this CTA's segment lies in [kWideMinLog2 / log2(e), 0], the
// per-token analogue of gamma >= 2^-0.75, so that the 128-token body's tile factors stay in
// range. Read by all threads of the CTA; the answer is uniform.
__device__ __forceinline__ bool gated_wide_ok(const Params& p, int bh, int tseg) {
    const int tbeg = tseg * p.seg_chunks * kC;
    const int tend = min(tbeg + p.seg_chunks * kC, p.N);
    const float* G = p.decay_in + (size_t)bh * p.N;
    int ok = 1;
#pragma unroll 4
    for (int t = tbeg + (int)threadIdx.x; t < tend; t += (int)blockDim.x) {
        const float g = G[t];
        ok &= (g <= 0.f && g * kLog2e >= kWideMinLog2) ? 1 : 0;
    }
    return __syncthreads_and(ok) != 0;
}

// STATE_ONLY: the first pass of a split sequence. Each CTA runs the state
// recurrence of one segment from a zero state (update products only; Q is not
// loaded and no output is formed) and writes the segment's end state U and total
// decay to the scratch buffers. seg_prefix_kernel then turns them into the
// segment start states S_in(g) = decay_{g-1} S_in(g-1) + U_{g-1}, S_in(0) =
// state_in, and the full pass starts each segment from its S_in.
// REV: the time-reversed direction, O_j = sum over later tokens i >= j of w_ij (q_j . k_i)
// v_i with the same weights (gamma^(i-j), or exp(G_i - G_j) for the gated form); the
// gradients dK and dV are such sums. The chunks are visited from the last back and the
// state is referenced at the token before the current chunk, R = sum_{i >= t0} w(i, t0-1)
// k_i^T v_i. With Gl the chunk's inclusive cumulative log-decay (L tokens) the factors
// mirror the forward's: key weights exp(Gl_i) instead of exp(Gl_{L-1} - Gl_i), cross-term
// row factors exp(Gl_{L-1} - Gl_j) instead of exp(Gl_j), the same chunk decay
// exp(Gl_{L-1}), and the upper triangle i >= j of the mask. Segments of a split sequence
// are chained from the last back too (blockIdx.z counts them from the end).
template <int DK, bool GATED, bool STATE_ONLY, bool REV>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, Params p) {
    // Launched as a programmatic dependent of the previous kernel in the stream: the CTAs
    // may be placed while that kernel drains, and wait here until it has completed and its
    // writes are visible, before any global memory is touched.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Heads with gamma close to 1, and gated segments whose every gate is that mild, take the
    // 128-token body (tc_wide.cuh); the choice is per CTA, so one launch serves a mix.
    if constexpr (wide_capable(DK, GATED, STATE_ONLY)) {
        if constexpr (GATED) {
            // the segment's place in time (the time-reversed form chains segments from the last)
            if (gated_wide_ok(p, blockIdx.y, REV ? p.units - 1 - (int)blockIdx.z : (int)blockIdx.z)) {
                wide_body<DK, REV, true>(tm_q, tm_k, tm_v, tm_o, p, 0.f);
                return;
            }
        } else {
            const float lgw = log2f(p.decay_in[blockIdx.y % p.H]);
            if (lgw >= kWideMinLog2 && lgw <= 0.f) {
                wide_body<DK, REV>(tm_q, tm_k, tm_v, tm_o, p, lgw);
                return;
            }
        }
    }
    using Lay = Layout<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int b) { return sbase + Lay::kBar + 8 * b; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::kTmemSlot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.x, bh = blockIdx.y;
    const int dv0 = slice * kDvS;
    const int seg = blockIdx.z;                                    // place in the chain of segments
    const int tseg = REV ? p.units - 1 - seg : seg;                // place in time
    const int cbase = tseg * p.seg_chunks;                         // first chunk of this segment
    const int nchunks = min(p.seg_chunks, (p.N + kC - 1) / kC - cbase);
    const bool last_seg = seg == p.units - 1;                      // the chain's last: writes state_out
    // token start of the i-th chunk visited (REV: from the segment's last chunk back)
    auto chunk_t0 = [&](int i) { return (cbase + (REV ? nchunks - 1 - i : i)) * kC; };
    if (STATE_ONLY && nchunks <= 0) {
        // REV only: a sub-segment past the end of a short last segment holds no tokens; its
        // local state is zero and its decay one
        float* so = p.seg_state + ((size_t)seg * gridDim.y + bh) * DK * p.dv + dv0;
        for (int e = threadIdx.x; e < DK * kDvS; e += blockDim.x) so[(size_t)(e / kDvS) * p.dv + e % kDvS] = 0.f;
        if (slice == 0 && threadIdx.x == 0) p.seg_ldec[(size_t)seg * gridDim.y + bh] = 0.f;
        return;
    }

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
    const float* G = GATED ? p.decay_in + (size_t)bh * p.N : nullptr;
    const float lg = GATED ? 0.f : log2f(p.decay_in[bh % p.H]);
    // Merged output accumulator (fixed gamma). With zeta'_j = gamma^(63-j), the decay mask
    // factors as gamma^(j-m) = zeta'_m / zeta'_j and the cross factor as gamma^(j+1) =
    // gamma^64 / zeta'_j, so
    //   O_j = (1 / zeta'_j) [ q_j (gamma^64 S) + sum_{m<=j} zeta'_m A_jm v_m ]
    // and both products accumulate into one TMEM region: the bf16 state copy holds
    // gamma^64 S, P holds zeta'_m A_jm, and the drain scales row j by 1 / zeta'_j. All
    // factors stay within [2^-64, 2^63] when gamma is in [1/2, 1], so nothing leaves the
    // normal range of bf16 or fp32 that the split form would keep; other gammas (and the
    // gated form) use the split accumulators. The choice is per CTA (one head).
    const bool merged = !GATED && !STATE_ONLY && lg >= -1.f && lg <= 0.f;
    const int nb = (DK <= 128 || merged) ? 2 : 1;  // attention buffers in use
    const int bcols = merged ? kC : 2 * kC;        // TMEM columns per attention buffer
    auto abuf = [&](int c) { return nb == 2 ? (c & 1) : 0; };   // attention buffer of chunk c
    auto ause = [&](int c) { return nb == 2 ? (c >> 1) : c; };  // how many chunks used that buffer before

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = -1;
            constexpr int NS = Lay::kStages;
            for (int i = 0; i < nchunks; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait(bar(kEmpty0 + s), ((i / NS) - 1) & 1, abort_flag)) break;
                const uint32_t st = sbase + Lay::kStage0 + s * Lay::kStageBytes;
                mbar_expect_tx(bar(kFull0 + s), STATE_ONLY ? Lay::kKBytes + Lay::kVBytes : Lay::kStageBytes);
                const int t0 = chunk_t0(i);
#pragma unroll
                for (int kb = 0; kb < DK / 64; ++kb) {
                    if (!STATE_ONLY) tma_load_3d(st + kb * kTile64, &tm_q, kb * 64, t0, bh, bar(kFull0 + s));
                    tma_load_3d(st + Lay::kQBytes + kb * kTile64, &tm_k, kb * 64, t0, bh, bar(kFull0 + s));
                }
                tma_load_3d(st + Lay::kQBytes + Lay::kKBytes, &tm_v, dv0, t0, bh, bar(kFull0 + s));
                tma_load_3d(st + Lay::kQBytes + Lay::kKBytes + kTile64, &tm_v, dv0 + 64, t0, bh, bar(kFull0 + s));
                issued = i;
            }
            if (*abort_flag && issued >= 0) {
                // drain the copies in flight before the CTA may exit
                for (int i = std::max(issued - NS + 1, 0); i <= issued; ++i)
                    mbar_drain(bar(kFull0 + i % NS), (i / NS) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc(64, kC, 0, 0);
            constexpr uint32_t id_oi = idesc(128, kC, 0, 0);
            constexpr uint32_t id_ov = idesc(128, kC, 1, 0);
            constexpr uint32_t id_up = idesc(128, DK, 1, 1);
            const uint32_t tS = tmem + Lay::kColS, tSop = tmem + Lay::kColSop;
            // A = Q K^T of chunk c into its attention buffer (both K-major, 128-byte swizzle,
            // 16-element K steps); the buffer is free once its previous chunk has been drained.
            auto issue_qk = [&](int c) {
                const int s = c % Lay::kStages, b = abuf(c);
                const uint32_t sQ = sbase + Lay::kStage0 + s * Lay::kStageBytes;
                const uint32_t sK = sQ + Lay::kQBytes;
                if (!mbar_wait(bar(kFull0 + s), (c / Lay::kStages) & 1, abort_flag)) return false;
                if (c >= nb && !mbar_wait(bar(kOFree0 + b), (ause(c) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t tA = tmem + Lay::kColA + bcols * b;
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kTile64 + (ks & 3) * 32;
                    mma_ss(tA, sdesc(sQ + off, 16, 1024), sdesc(sK + off, 16, 1024), id_qk, ks > 0);
                }
                mma_commit(bar(kAFull0 + b));
                return true;
            };
            const bool primed = STATE_ONLY || nb == 1 || nchunks == 0 || issue_qk(0);
            for (int i = 0; primed && i < nchunks; ++i) {
                const int s = i % Lay::kStages, z = i & 1, b = abuf(i);  // TMA stage, ZV buffer, attention buffer
                const uint32_t sQ = sbase + Lay::kStage0 + s * Lay::kStageBytes;
                const uint32_t sK = sQ + Lay::kQBytes;
                const uint32_t sV = sK + Lay::kKBytes;
                const uint32_t sZV = sbase + Lay::kZV + z * Lay::kVBytes;
                // merged: both output products add into the Q K^T columns; split: O_intra has its own
                const uint32_t tA = tmem + Lay::kColA + bcols * b, tO = merged ? tA : tA + kC;
                const uint32_t sP = sbase + Lay::kP + b * kTile64;
                if (STATE_ONLY) {
                    if (!mbar_wait(bar(kFull0 + s), (i / Lay::kStages) & 1, abort_flag)) break;
                    if (!mbar_wait(bar(kZV0 + z), (i >> 1) & 1, abort_flag) ||
                        !mbar_wait(bar(kSReady), i & 1, abort_flag))
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kC / 16; ++ks)
                        mma_ss(tS, sdesc(sZV + ks * 2048, kTile64, 1024), sdesc(sK + ks * 2048, kTile64, 1024), id_up, 1);
                    mma_commit(bar(kSFull));
                    mma_commit(bar(kEmpty0 + s));
                    continue;
                }
                // Issue order. The state round trip (the state epilogue reads S_i and writes the
                // next bf16 copy) is the loop-carried chain, so the products it waits for go first
                // and are committed on their own: update(i), O_inter(i) -> kSFull. The rest of the
                // chunk's tensor work -- the next chunk's Q K^T (two buffers) and O_intra(i) --
                // then runs in the pipe while the round trip is under way.
                if (nb == 1 && !issue_qk(i)) break;
                if (!mbar_wait(bar(kZV0 + z), (i >> 1) & 1, abort_flag) || !mbar_wait(bar(kSReady), i & 1, abort_flag))
                    break;
                tc_fence_after();
                // S^T += (zeta V)^T K: A = ZV MN-major, B = K tile MN-major (dk blocks 8 KB apart)
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_ss(tS, sdesc(sZV + ks * 2048, kTile64, 1024), sdesc(sK + ks * 2048, kTile64, 1024), id_up, 1);
                // O_inter^T = S_op^T Q^T into the same TMEM columns as Q K^T: only needs the
                // epilogue to have read Q K^T, not to have finished P.
                if (!mbar_wait(bar(kARead0 + b), ause(i) & 1, abort_flag)) break;
                tc_fence_after();
                // A from TMEM (bf16 pairs per column), B = Q tile K-major
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kTile64 + (ks & 3) * 32;
                    mma_ts(tA, tSop + ks * 8, sdesc(sQ + off, 16, 1024), id_oi, ks > 0);
                }
                // S_i is final and the cross term has read S_op: the state epilogue may now
                // overwrite S_op and decay S.
                mma_commit(bar(kSFull));
                if (nb == 2 && i + 1 < nchunks && !issue_qk(i + 1)) break;
                if (!mbar_wait(bar(kPReady0 + b), ause(i) & 1, abort_flag)) break;
                tc_fence_after();
                // O_intra^T = V^T P^T: A = V tile MN-major (dv blocks 8 KB apart), B = P K-major
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_ss(tO, sdesc(sV + ks * 2048, kTile64, 1024), sdesc(sP + ks * 32, 16, 1024), id_ov,
                           merged || ks > 0);
                mma_commit(bar(kOFull0 + b));
                mma_commit(bar(kEmpty0 + s));
            }
            // every issued MMA must complete before TMEM can be released
            mma_commit(bar(kDrain));
            mbar_drain(bar(kDrain), 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ attention epilogue (warps 2..5)
      if (!STATE_ONLY) {
        const int te = threadIdx.x - 64;          // 0..127
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float* cum = reinterpret_cast<float*>(sm + Lay::kAgTab);  // gated: in-chunk cumsum (log2 units), per buffer
        float* rr = cum + 2 * kC;  // row factor of the drain, per buffer: r_j (split), 1 / zeta'_j (merged)
        float* pw = rr + 2 * kC;                                  // fixed gamma: gamma^t, t = 0..64
        float* gcol = pw;  // gated (pw unused): column factors [64] of the current chunk, then max |c|
        auto wait_all = [&](int b, uint32_t parity) {  // every thread reaches the barrier; uniform result
            mbar_wait(bar(b), parity, abort_flag);
            group_sync(1);
            return *abort_flag == 0;
        };
        // row factors of the drain: per buffer where they depend on the chunk (gated; REV
        // split, whose factor gamma^(L-1-j) depends on the chunk's length), else one table
        constexpr bool kRowPerChunk = GATED || REV;
        if (!GATED) {
            if (te <= kC) pw[te] = pow_int_log2(lg, te);
            group_sync(1);
            if (te < kC) rr[te] = merged ? pow_int_log2(-lg, REV ? te : kC - 1 - te) : pw[te + 1];
        }
        // gated: the next chunk's gates, prefetched by the first warp as they are in memory and
        // scaled to log2 units only where the chunk's scan reads them, so that no instruction
        // waits for the load before the group barrier
        float g0 = 0.f, g1 = 0.f;
        if (GATED && te < 32) {
            const int a = chunk_t0(0) + 2 * te;
            g0 = a < p.N ? G[a] : 0.f;
            g1 = a + 1 < p.N ? G[a + 1] : 0.f;
        }
        // ---------------- P = mask(Q K^T) of chunk c in bf16 (its attention buffer): row j, 32 columns per thread
        auto do_p = [&](int ci) {
            const int b = abuf(ci);
            const int t0 = chunk_t0(ci);
            float* cumb = cum + b * kC;
            if (GATED) {
                if (te < 32) {
                    warp_cumsum64(g0 * kLog2e, g1 * kLog2e, lane, cumb);
                    // largest |cumulative log2-decay| of the chunk (this lane's two values, just written)
                    float mx = fmaxf(fabsf(cumb[2 * lane]), fabsf(cumb[2 * lane + 1]));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    if (lane == 0) gcol[kC] = mx;
                    // prefetch the next chunk's gates (none past the last chunk: a >= N reads zero)
                    const int a = (ci + 1 < nchunks ? chunk_t0(ci + 1) : p.N) + 2 * te;
                    g0 = a < p.N ? G[a] : 0.f;
                    g1 = a + 1 < p.N ? G[a + 1] : 0.f;
                }
                group_sync(1);
                // forward exp(Gl_j); REV exp(Gl_last - Gl_j) (gates past N are zero, so Gl_63 = Gl_{L-1})
                if (te < kC) rr[b * kC + te] = exp2f(REV ? cumb[kC - 1] - cumb[te] : cumb[te]);
                // column factors of the weights exp2(c_j - c_m) = exp2(c_j) exp2(-c_m) (REV: the
                // mirror), used when every |c| of the chunk is at most 100 so that both factors
                // and their products with Q K^T stay inside the fp32 range
                if (te < kC) gcol[te] = exp2f(REV ? cumb[te] : -cumb[te]);
            } else if (REV && !merged) {
                const int L = min(kC, p.N - t0);
                if (te < kC) rr[b * kC + te] = te < L ? pw[L - 1 - te] : 0.f;
            }
            if (!wait_all(kAFull0 + b, ause(ci) & 1)) return false;
            tc_fence_after();
            {
                uint32_t a[32];
                tmem_ld16x2(tmem + lane_off + Lay::kColA + bcols * b, a);
                const int j = quarter * 16 + (lane & 15);  // M=64 accumulator: row j in lane 32*(j/16) + j%16
                const int m0 = (lane >> 4) * 32;
                // all table reads before any shared-memory store (the pointers may alias)
                float w[32];
                if (GATED) {
                    const float cj = cumb[j];
                    if (gcol[kC] <= 100.f) {  // uniform over the group: one value per chunk
                        const float rj = exp2f(REV ? -cj : cj);
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int m = m0 + c;
                            w[c] = (REV ? m < j : m > j) ? 0.f : (m == j ? 1.f : gcol[m] * rj);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) w[c] = REV ? cumb[m0 + c] - cj : cj - cumb[m0 + c];
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int m = m0 + c;
                            w[c] = (REV ? m < j : m > j) ? 0.f : (m == j ? 1.f : exp2f(w[c]));
                        }
                    }
                } else if (REV) {
                    // split: gamma^(m-j); merged: zeta'_m = gamma^m
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int m = m0 + c;
                        w[c] = m < j ? 0.f : pw[merged ? m : m - j];
                    }
                } else {
                    // split: gamma^(j-m); merged: zeta'_m = gamma^(63-m)
                    const int base = merged ? kC - 1 : j;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int m = m0 + c;
                        w[c] = m > j ? 0.f : pw[base - m];
                    }
                }
                tmem_wait_ld();
                // Q K^T is in registers: the cross-term product may overwrite those columns now
                tc_fence_before();
                group_sync(1);
                if (te == 0) mbar_arrive(bar(kARead0 + b));
                uint32_t u[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    u[c] = pack_bf16(__uint_as_float(a[2 * c]) * w[2 * c], __uint_as_float(a[2 * c + 1]) * w[2 * c + 1]);
                uint8_t* prow = sm + Lay::kP + b * kTile64 + j * 128;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int chunk16 = (m0 >> 3) + cc;
                    *reinterpret_cast<uint4*>(prow + ((chunk16 ^ (j & 7)) << 4)) =
                        make_uint4(u[4 * cc], u[4 * cc + 1], u[4 * cc + 2], u[4 * cc + 3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync(1);
            if (te == 0) mbar_arrive(bar(kPReady0 + b));
            return true;
        };
        // ---------------- O = O_intra + r_j O_inter of chunk c -> bf16 -> staging -> TMA store
        auto do_drain = [&](int ci) {
            const int b = abuf(ci);
            const int t0 = chunk_t0(ci);
            const float* rrb = (kRowPerChunk && (GATED || !merged)) ? rr + b * kC : rr;
            const uint32_t tA = tmem + lane_off + Lay::kColA + bcols * b;
            if (te == 0) tma_store_wait_read();  // the previous chunk's O store has read the staging tile
            if (!wait_all(kOFull0 + b, ause(ci) & 1)) return false;
            tc_fence_after();
            {
                // The output accumulators read as 16-lane x 8-column fragments: lanes quarter*32 +
                // 16 hf + {g, g + 8} (g = lane / 4), token columns 8k + 2 (lane % 4) + {0, 1}, i.e.
                // pairs of adjacent tokens of one dv column, which stmatrix .trans writes as 8 x 8
                // blocks of (token rows x dv columns) into the two staging boxes (dv halves).
                // All of them are read before the TMEM columns are released to the next chunk.
                uint32_t zi[2][32], ze[2][32];  // merged: the one accumulator; split: O_intra, O_inter
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t lh = (uint32_t)(16 * hf) << 16;
                    tmem_ld16x256b_x8(tA + lh + (merged ? 0 : kC), zi[hf]);
                    if (!merged) tmem_ld16x256b_x8(tA + lh, ze[hf]);
                }
                tmem_wait_ld();
                tc_fence_before();
                group_sync(1);
                if (te == 0) mbar_arrive(bar(kOFree0 + b));
                const int i2 = 2 * (lane & 3), bk = lane >> 3, q = lane & 7;
#pragma unroll
                for (int k = 0; k < 8; k += 2) {
                    // row factors of tokens 8k' + i2 + {0, 1}, k' = k, k + 1 (read before any shared store)
                    const float2 f0 = reinterpret_cast<const float2*>(rrb)[(8 * k + i2) >> 1];
                    const float2 f1 = reinterpret_cast<const float2*>(rrb)[(8 * k + 8 + i2) >> 1];
                    const int jr = 8 * (k + (bk >> 1)) + q;  // token row of the block row this lane addresses
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float f = e < 4 ? ((e & 1) ? f0.y : f0.x) : ((e & 1) ? f1.y : f1.x);
                            const float a = __uint_as_float(zi[hf][4 * k + e]);
                            o[e] = merged ? f * a : fmaf(f, __uint_as_float(ze[hf][4 * k + e]), a);
                        }
                        const int dvb = quarter * 32 + 16 * hf + 8 * (bk & 1);  // first dv column of the block
                        const uint32_t box = sbase + Lay::kOst + (dvb >> 6) * kTile64;
                        stmatrix_x4_trans(box + jr * 128 + ((((dvb & 63) >> 3) ^ (jr & 7)) << 4), pack_bf16(o[0], o[1]),
                                          pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
                    }
                }
            }
            fence_proxy_async();
            group_sync(1);
            if (te == 0) {
                tma_out_3d(p.o_add, &tm_o, dv0, t0, bh, sbase + Lay::kOst);
                tma_out_3d(p.o_add, &tm_o, dv0 + 64, t0, bh, sbase + Lay::kOst + kTile64);
                tma_store_commit();
            }
            return true;
        };
        // With two buffers the mask of chunk i+1 is built while chunk i's output products run,
        // then chunk i is drained; with one buffer the chunks go mask, drain, mask, drain.
        if (nb == 2) {
            bool ok = nchunks == 0 || do_p(0);
            for (int i = 0; ok && i < nchunks; ++i) {
                if (i + 1 < nchunks) ok = do_p(i + 1);
                ok = ok && do_drain(i);
            }
        } else {
            for (int i = 0; i < nchunks; ++i)
                if (!do_p(i) || !do_drain(i)) break;
        }
        if (te == 0) tma_store_wait_all();
      }
    } else {
        // ------------------------------------------------------------ state epilogue (warps 6..9)
        const int ts = threadIdx.x - 192;         // 0..127
        const int quarter = warp & 3;
        const int d = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float* cum = reinterpret_cast<float*>(sm + Lay::kSgTab);
        float* zeta = cum + kC;
        float* dec = zeta + kC;
        auto wait_all = [&](int b, uint32_t parity) {
            mbar_wait(bar(b), parity, abort_flag);
            group_sync(2);
            return *abort_flag == 0;
        };
        float g0 = 0.f, g1 = 0.f;  // gated: the next chunk's gates, prefetched as in the attention group
        if (GATED && ts < 32) {
            const int a = chunk_t0(0) + 2 * ts;
            g0 = a < p.N ? G[a] : 0.f;
            g1 = a + 1 < p.N ? G[a + 1] : 0.f;
        }
        float ldec_sum = 0.f;  // log2 of the decay accumulated over this segment
        // Lazy decay. The state is held as S_i = c_i * T_i with T in TMEM and the scalar c_i in
        // a register: the update adds (zeta V / c_{i+1}) onto T, and T is rewritten only when
        // c would drop below kRenorm (then T <- c_i d_{i+1} T_i and c_{i+1} = 1). This keeps the
        // per-chunk round trip to one read of T and one write of the bf16 copy.
        constexpr float kRenorm = 9.094947e-13f;  // 2^-40
        // zeta-scaled V of chunk c into ZV buffer c & 1, divided by the scale c_{next} that
        // make_zv picks from c_prev (the current scale) and the chunk's decay.
        auto make_zv = [&](int c, float c_prev, bool force_renorm, float& decay, bool& renorm, float& c_next) {
            const int t0 = chunk_t0(c), L = min(kC, p.N - t0);
            if (GATED) {
                if (ts < 32) {
                    warp_cumsum64(g0 * kLog2e, g1 * kLog2e, lane, cum);
                    const int a = (c + 1 < nchunks ? chunk_t0(c + 1) : p.N) + 2 * ts;
                    g0 = a < p.N ? G[a] : 0.f;
                    g1 = a + 1 < p.N ? G[a + 1] : 0.f;
                }
                group_sync(2);
                if (ts < kC) zeta[ts] = ts < L ? exp2f(REV ? cum[ts] : cum[L - 1] - cum[ts]) : 0.f;
                if (ts == 0) {
                    dec[0] = exp2f(cum[L - 1]);
                    dec[1] = cum[L - 1];
                }
            } else {
                if (ts < kC) zeta[ts] = ts < L ? pow_int_log2(lg, REV ? ts + 1 : L - 1 - ts) : 0.f;
                if (ts == 0) {
                    dec[0] = pow_int_log2(lg, L);
                    dec[1] = lg * (float)L;
                }
            }
            if (!wait_all(kFull0 + c % Lay::kStages, (c / Lay::kStages) & 1)) return false;  // V tile of chunk c landed
            decay = dec[0];
            ldec_sum += dec[1];
            renorm = force_renorm || !(c_prev * decay >= kRenorm);
            c_next = renorm ? 1.f : c_prev * decay;
            const float inv = 1.f / c_next;
            const uint8_t* vt = sm + Lay::kStage0 + (c % Lay::kStages) * Lay::kStageBytes + Lay::kQBytes + Lay::kKBytes;
            uint8_t* zv = sm + Lay::kZV + (c & 1) * Lay::kVBytes;
            // 16-byte chunks ci = e * 128 + ts; the swizzle stays inside a 128-byte row, so the
            // row (token) of a chunk is (ci mod 512) / 8. All loads before any store (aliasing).
            uint4 x[8];
            float z[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int ci = e * kEpiThreads + ts;
                z[e] = zeta[(ci & 511) >> 3] * inv;
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
            for (int e = 0; e < 8; ++e) *reinterpret_cast<uint4*>(zv + (e * kEpiThreads + ts) * 16) = x[e];
            fence_proxy_async();
            group_sync(2);
            if (ts == 0) mbar_arrive(bar(kZV0 + (c & 1)));
            return true;
        };

        // The bf16 state copy feeding chunk c's cross term is S (split output accumulators)
        // or, merged, gamma^64 S (forward) or gamma^(L_c - 1) S (REV, L_c the chunk's length).
        auto sop_of = [&](int c) {
            return !merged ? 1.f : REV ? pow_int_log2(lg, min(kC, p.N - chunk_t0(c)) - 1) : pow_int_log2(lg, kC);
        };
        const float sop = sop_of(0);
        float dec0 = 0.f, c_cur = 1.f;
        bool renorm = true;
        bool ok = make_zv(0, 1.f, true, dec0, renorm, c_cur);
        if (ok) {
            // initial state: S_op = bf16(sop S_in), T = decay_0 * S_in, c = 1. The state-only pass
            // starts from zero; the full pass from segment_start_state().
            const float* sin = STATE_ONLY ? nullptr : segment_start_state(p, seg, bh, DK, dv0 + d);
#pragma unroll 1
            for (int cb = 0; cb < DK / 32; ++cb) {
                uint32_t w[32], h[16];
#pragma unroll
                for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(sin ? sin[(size_t)(cb * 32 + c) * p.dv] : 0.f);
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    h[c] = pack_bf16(__uint_as_float(w[2 * c]) * sop, __uint_as_float(w[2 * c + 1]) * sop);
#pragma unroll
                for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(__uint_as_float(w[c]) * dec0);
                tmem_st32(tmem + lane_off + Lay::kColS + cb * 32, w);
                tmem_st16(tmem + lane_off + Lay::kColSop + cb * 16, h);
            }
            tmem_wait_st();
            tc_fence_before();
            group_sync(2);
            if (ts == 0) mbar_arrive(bar(kSReady));
        }
        for (int i = 0; i < nchunks && ok; ++i) {
            const bool last = (i == nchunks - 1);
            float dec_next = 0.f, c_next = 1.f;
            // the next chunk's zeta V is ready before this chunk's state update completes
            if (!last && !make_zv(i + 1, c_cur, false, dec_next, renorm, c_next)) break;
            if (!wait_all(kSFull, i & 1)) break;
            tc_fence_after();
            if (last) {
                float* so = nullptr;
                if (STATE_ONLY) {
                    so = p.seg_state + ((size_t)seg * gridDim.y + bh) * DK * p.dv + dv0 + d;
                    if (slice == 0 && ts == 0) p.seg_ldec[(size_t)seg * gridDim.y + bh] = ldec_sum;
                } else if (last_seg) {
                    so = p.state_out;
                    if (so) so += ((size_t)bh * DK) * p.dv + dv0 + d;
                }
                if (so) {
#pragma unroll 1
                    for (int cb = 0; cb < DK / 32; ++cb) {
                        uint32_t w[32];
                        tmem_ld32(tmem + lane_off + Lay::kColS + cb * 32, w);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) so[(size_t)(cb * 32 + c) * p.dv] = __uint_as_float(w[c]) * c_cur;
                    }
                }
            } else if (!STATE_ONLY || renorm) {
                // S_op = bf16(sop c_i T_i) for the next cross term; on renormalisation also
                // T <- c_i d_{i+1} T_i so that the next update (scaled by 1/c_{i+1} = 1) adds onto it.
                // The state-only pass needs no S_op and touches T only to renormalise.
                const float tscale = c_cur * dec_next, hscale = c_cur * sop_of(i + 1);
#pragma unroll 1
                for (int cb = 0; cb < DK / 64; ++cb) {
                    uint32_t w0[32], w1[32], h[16];
                    tmem_ld32(tmem + lane_off + Lay::kColS + cb * 64, w0);
                    tmem_ld32(tmem + lane_off + Lay::kColS + cb * 64 + 32, w1);
                    tmem_wait_ld();
                    if (!STATE_ONLY) {
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            h[c] = pack_bf16(__uint_as_float(w0[2 * c]) * hscale, __uint_as_float(w0[2 * c + 1]) * hscale);
                        tmem_st16(tmem + lane_off + Lay::kColSop + cb * 32, h);
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            h[c] = pack_bf16(__uint_as_float(w1[2 * c]) * hscale, __uint_as_float(w1[2 * c + 1]) * hscale);
                        tmem_st16(tmem + lane_off + Lay::kColSop + cb * 32 + 16, h);
                    }
                    if (renorm) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            w0[c] = __float_as_uint(__uint_as_float(w0[c]) * tscale);
                            w1[c] = __float_as_uint(__uint_as_float(w1[c]) * tscale);
                        }
                        tmem_st32(tmem + lane_off + Lay::kColS + cb * 64, w0);
                        tmem_st32(tmem + lane_off + Lay::kColS + cb * 64 + 32, w1);
                    }
                }
                tmem_wait_st();
            }
            if (!last) {
                tc_fence_before();
                group_sync(2);
                if (ts == 0) mbar_arrive(bar(kSReady));
                c_cur = c_next;
            }
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

constexpr int kMaxSegments = 16;  // segments of a split sequence, at most

// Segment start states of a split sequence, between the two passes: seg_state[g] holds
// U_g (segment g's end state from a zero start) on entry and S_in(g + 1) = Gamma_g S_in(g)
// + U_g on exit, with S_in(0) = state_in (or zero) and Gamma_g = 2^seg_ldec[g]. One thread
// per 4 consecutive state elements (no grid-stride loop: the kernel is latency-bound, so
// every thread issues its NS loads at once and the grid covers the states in one pass);
// NS = G - 1 states is a template argument so that exactly those loads are in flight.
// Every full-pass CTA then reads one state instead of folding all earlier segments
// itself. seg_state is the library's scratch (16-byte aligned); state_in is read element
// by element (only 4-byte alignment is required of it).
template <int NS>
__global__ void __launch_bounds__(256)
seg_prefix_kernel(const float* __restrict__ state_in, float* __restrict__ seg_state, const float* __restrict__ seg_ldec,
                  int BH, int per_bh) {
    const size_t n4 = (size_t)BH * per_bh / 4;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const int bh = (int)(i * 4 / per_bh);
    float4 u[NS];
    float gam[NS];
#pragma unroll
    for (int g = 0; g < NS; ++g) {
        u[g] = __ldcs(reinterpret_cast<const float4*>(seg_state + (size_t)g * BH * per_bh) + i);
        gam[g] = seg_ldec[(size_t)g * BH + bh];
    }
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in) x = make_float4(state_in[4 * i], state_in[4 * i + 1], state_in[4 * i + 2], state_in[4 * i + 3]);
#pragma unroll
    for (int g = 0; g < NS; ++g) {
        const float d = exp2f(gam[g]);
        x = make_float4(fmaf(d, x.x, u[g].x), fmaf(d, x.y, u[g].y), fmaf(d, x.z, u[g].z), fmaf(d, x.w, u[g].w));
        reinterpret_cast<float4*>(seg_state + (size_t)g * BH * per_bh)[i] = x;
    }
}

template <int NS>
inline void launch_seg_prefix_n(const float* state_in, float* seg_state, const float* seg_ldec, int BH, int per_bh,
                                unsigned blocks, cudaStream_t st) {
    seg_prefix_kernel<NS><<<blocks, 256, 0, st>>>(state_in, seg_state, seg_ldec, BH, per_bh);
}

// Launches the prefix over `ns` segment states (1 <= ns < kMaxSegments).
inline cudaError_t launch_seg_prefix(const float* state_in, float* seg_state, const float* seg_ldec, int ns, int BH,
                                     int per_bh, cudaStream_t st) {
    const size_t n4 = (size_t)BH * per_bh / 4;
    const unsigned blocks = (unsigned)((n4 + 255) / 256);
    switch (ns) {
        case 1: launch_seg_prefix_n<1>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 2: launch_seg_prefix_n<2>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 3: launch_seg_prefix_n<3>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 4: launch_seg_prefix_n<4>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 5: launch_seg_prefix_n<5>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 6: launch_seg_prefix_n<6>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 7: launch_seg_prefix_n<7>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 8: launch_seg_prefix_n<8>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 9: launch_seg_prefix_n<9>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 10: launch_seg_prefix_n<10>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 11: launch_seg_prefix_n<11>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 12: launch_seg_prefix_n<12>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 13: launch_seg_prefix_n<13>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 14: launch_seg_prefix_n<14>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        case 15: launch_seg_prefix_n<15>(state_in, seg_state, seg_ldec, BH, per_bh, blocks, st); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// Self-test of the failure path: one CTA takes TMEM like the chunk kernels, waits with
// their bounded wait on an mbarrier that nothing completes, takes the timeout path (device
// error word, abort flag), releases TMEM and returns. Nothing faults or hangs.
__global__ void __launch_bounds__(64, 1) selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ uint32_t slot;
    __shared__ int abort_storage;
    const uint32_t b = smem_u32(&bar_storage);
    volatile int* abort_flag = &abort_storage;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&slot)), "r"(32)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = slot;
    if (threadIdx.x == 0) mbar_wait(b, 0, abort_flag, limit_ns);  // nothing arrives: runs out
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(32) : "memory");
    }
}

// ------------------------------------------------------------------ host side

// Per-device facts the host code needs on every call, cached per device (a process may
// drive several GPUs from several threads). Racing first lookups store the same value,
// so plain atomics suffice.
constexpr int kMaxDevices = 64;

inline int current_device() {
    int dev = 0;
    return (cudaGetDevice(&dev) == cudaSuccess && dev >= 0) ? dev : -1;
}

// 1 if the current device is sm_100 (the tensor-core path's target), else 0.
inline bool tc_device_ok() {
    static std::atomic<int> cached[kMaxDevices];  // 0 = unknown, 1 = yes, 2 = no
    const int dev = current_device();
    if (dev < 0) return false;
    auto query = [dev] {
        int major = 0, minor = 0;
        return cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
               cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
               major == 10 && minor == 0;
    };
    if (dev >= kMaxDevices) return query();
    int c = cached[dev].load(std::memory_order_relaxed);
    if (c == 0) {
        c = query() ? 1 : 2;
        cached[dev].store(c, std::memory_order_relaxed);
    }
    return c == 1;
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3D bf16 map over [BH][N][inner] with a 64 x 64 box and 128-byte swizzle. Rows are
// ld elements apart (ld = 0: dense, ld = inner), so a column slice of a wider tensor
// can be read in place.
inline bool make_map(CUtensorMap* m, const void* base, int inner, int N, int BH, int ld = 0) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t row = (cuuint64_t)(ld ? ld : inner);
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {row * 2, row * 2 * N};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc

inline bool tc_chunk_supported(int dk, int dv, int chunk, bool bf16) {
    return bf16 && (dk == 64 || dk == 128 || dk == 256) && dv % tc::kDvS == 0 && chunk % tc::kC == 0 &&
           tc::tc_device_ok();
}

namespace tc {

// Streaming multiprocessors of the current device (148 on a B200 if the query fails).
inline int sm_count() {
    static std::atomic<int> cached[kMaxDevices];
    const int dev = current_device();
    auto query = [dev] {
        int n = 0;
        if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        return n;
    };
    if (dev < 0 || dev >= kMaxDevices) return query();
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        n = query();
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Sequence split: with few (head, dv-slice) CTAs the sequence is cut into G
// segments so that about one CTA per SM runs. Segments are whole chunks.
struct Plan {
    int G;           // segments
    int seg_chunks;  // chunks per segment
    int F;           // state-only sub-segments per segment (seg_chunks / F chunks each)
    int subs() const { return F * (G - 1); }  // sub-segments whose end states the state-only pass writes
};

// sub_segments = false keeps one state-only CTA per segment (less scratch). concurrent:
// how many launches of this shape the caller runs at the same time on other streams
// (their CTAs count towards filling the SMs).
inline Plan plan(int B, int H, int N, int dv, bool sub_segments = true, int concurrent = 1) {
    const int ctas = B * H * (dv / kDvS) * concurrent;
    const int nchunks = (N + kC - 1) / kC;
    int G = 1;
    if (2 * ctas <= sm_count()) G = std::min(std::min(sm_count() / ctas, kMaxSegments), nchunks / 4);
    if (G < 2) return {1, nchunks, 1};
    // an even number of 64-token chunks, so that 128-token tiles do not straddle segments
    const int seg_chunks = ((nchunks + G - 1) / G + 1) & ~1;
    G = (nchunks + seg_chunks - 1) / seg_chunks;
    // Only segments 0..G-2 need end states, so the state-only pass would leave SMs idle: cut
    // each of those segments into F sub-segments while that still fits the SMs.
    int F = 1;
    if (sub_segments)
        while (2 * F * ctas * (G - 1) <= sm_count() && seg_chunks % (2 * F) == 0 && 2 * F * (G - 1) < kMaxSegments) F *= 2;
    return {G, seg_chunks, F};
}

// Scratch of a split sequence: end states [F(G-1), BH, dk, dv] fp32, log2 decays [F(G-1), BH],
// and, when state_in and state_out are the same buffer, a copy of state_in (every segment
// reads state_in while the last one writes state_out, so they must not share memory).
inline size_t scratch_states_bytes(const Plan& pl, int BH, int dk, int dv) {
    return sizeof(float) * (size_t)pl.subs() * BH * dk * dv;
}
inline size_t scratch_ldec_bytes(const Plan& pl, int BH) {
    return (sizeof(float) * (size_t)pl.subs() * BH + 255) & ~size_t(255);
}
inline size_t scratch_bytes(const Plan& pl, int BH, int dk, int dv, bool alias) {
    if (pl.G < 2) return 0;
    return scratch_states_bytes(pl, BH, dk, dv) + scratch_ldec_bytes(pl, BH) +
           (alias ? sizeof(float) * (size_t)BH * dk * dv : 0);
}

// Dynamic shared memory of one instantiation: the 64-token layout, or the 128-token one
// where the kernel may run that body.
template <int DK, bool GATED, bool STATE_ONLY>
constexpr int kernel_smem() {
    if constexpr (wide_capable(DK, GATED, STATE_ONLY))
        return std::max(Layout<DK>::kSmemAlloc, WideLayout<DK>::kSmemAlloc);
    else
        return Layout<DK>::kSmemAlloc;
}

// Launches a tensor-core kernel with programmatic stream serialization: its CTAs may start
// while the previous kernel in the stream finishes, and wait (griddepcontrol.wait, the
// kernel's first instruction) until that kernel has completed.
template <typename... P, typename... A>
inline cudaError_t launch_dependent(void (*kernel)(P...), dim3 grid, int threads, size_t smem, cudaStream_t st,
                                    A&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

template <int DK, bool GATED, bool REV>
ret_status launch_dk(const void* q, const void* k, const void* v, const float* decay, void* o,
                     const float* state_in, float* state_out, int B, int H, int N, int dv, const Plan& pl,
                     void* scratch, cudaStream_t st, int ldq, int ldk, bool o_add) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, DK, N, BH, ldq) || !make_map(&mk, k, DK, N, BH, ldk) || !make_map(&mv, v, dv, N, BH) ||
        !make_map(&mo, o, dv, N, BH))
        return RET_ERR_CUDA;
    Params prm{decay, state_in, state_out, nullptr, nullptr, H, N, dv, pl.seg_chunks, pl.F, pl.G, o_add ? 1 : 0};
    if (pl.G > 1) {
        uint8_t* sc = static_cast<uint8_t*>(scratch);
        prm.seg_state = reinterpret_cast<float*>(sc);
        prm.seg_ldec = reinterpret_cast<float*>(sc + scratch_states_bytes(pl, BH, DK, dv));
        if (state_in && state_in == state_out) {
            float* copy = reinterpret_cast<float*>(sc + scratch_states_bytes(pl, BH, DK, dv) + scratch_ldec_bytes(pl, BH));
            if (cudaMemcpyAsync(copy, state_in, sizeof(float) * (size_t)BH * DK * dv, cudaMemcpyDeviceToDevice, st) !=
                cudaSuccess)
                return RET_ERR_CUDA;
            prm.state_in = copy;
        }
        auto k1 = state_tc_kernel<DK, GATED, REV>;
        constexpr int smem1 = StateLayout<DK, state_tile(GATED)>::kSmemAlloc;
        if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1) != cudaSuccess)
            return RET_ERR_CUDA;
        Params prm1 = prm;  // the state-only pass runs over the sub-segments
        prm1.seg_chunks = pl.seg_chunks / pl.F;
        prm1.units = pl.F * pl.G;
        if (launch_dependent(k1, dim3(dv / kDvS, BH, pl.subs()), kSThreads, smem1, st, mk, mv, prm1) != cudaSuccess)
            return RET_ERR_CUDA;
        if (launch_seg_prefix(prm.state_in, prm.seg_state, prm.seg_ldec, pl.subs(), BH, DK * dv, st) != cudaSuccess)
            return RET_ERR_CUDA;
    }
    auto k2 = chunk_tc_kernel<DK, GATED, false, REV>;
    constexpr int smem2 = kernel_smem<DK, GATED, false>();
    if (cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2) != cudaSuccess)
        return RET_ERR_CUDA;
    return launch_dependent(k2, dim3(dv / kDvS, BH, pl.G), kThreads, smem2, st, mq, mk, mv, mo, prm) == cudaSuccess ? RET_OK
                                                                                                     : RET_ERR_CUDA;
}

// Runs the tensor-core path with caller-provided scratch (at least scratch_bytes()).
// ldq, ldk: row strides of q and k in elements (0: dense rows of dk). REV: the
// time-reversed direction (sums over later tokens), see chunk_tc_kernel. o_add: add the
// output onto o instead of storing it.
template <bool GATED, bool REV = false>
ret_status launch_with_scratch(const void* q, const void* k, const void* v, const float* decay, void* o,
                               const float* state_in, float* state_out, int B, int H, int N, int dk, int dv,
                               const Plan& pl, void* scratch, cudaStream_t st, int ldq = 0, int ldk = 0,
                               bool o_add = false) {
    switch (dk) {
        case 64:
            return launch_dk<64, GATED, REV>(q, k, v, decay, o, state_in, state_out, B, H, N, dv, pl, scratch, st,
                                             ldq, ldk, o_add);
        case 128:
            return launch_dk<128, GATED, REV>(q, k, v, decay, o, state_in, state_out, B, H, N, dv, pl, scratch, st,
                                              ldq, ldk, o_add);
        case 256:
            return launch_dk<256, GATED, REV>(q, k, v, decay, o, state_in, state_out, B, H, N, dv, pl, scratch, st,
                                              ldq, ldk, o_add);
    }
    return RET_ERR_UNSUPPORTED;
}

}  // namespace tc

inline int tc_chunk_launches(int B, int H, int N, int, int dv, int concurrent = 1) {
    return tc::plan(B, H, N, dv, true, concurrent).G > 1 ? 3 : 1;
}

namespace tc {

// The default stream-ordered pool of a device returns its memory to the system
// at every synchronisation unless its release threshold is raised; then each
// call would map fresh memory. Raise it once per device so that repeated calls
// reuse the pool's memory.
inline void keep_pool_memory() {
    static std::atomic<bool> done[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices || done[dev].exchange(true)) return;
    cudaMemPool_t pool;
    if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
        uint64_t threshold = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &threshold);
    }
}

// End state of a whole sequence from a zero start, without outputs: the state-only kernel
// over `subs` sub-segments of sub_chunks chunks (enough CTAs to fill the SMs), combined by
// seg_prefix_kernel; with one sub-segment it writes state_out directly. Scratch: the
// sub-segments' states (only when subs > 1) and their log2 decays.
inline void state_plan(int B, int H, int N, int dv, int& subs, int& sub_chunks) {
    const int ctas = B * H * (dv / kDvS);
    const int nchunks = (N + kC - 1) / kC;
    subs = std::max(1, std::min(std::min(sm_count() / ctas, kMaxSegments - 1), nchunks));
    sub_chunks = (nchunks + subs - 1) / subs;
    subs = (nchunks + sub_chunks - 1) / sub_chunks;
}
inline size_t state_scratch_bytes(int subs, int BH, int dk, int dv) {
    return (subs > 1 ? sizeof(float) * (size_t)subs * BH * dk * dv : 0) +
           ((sizeof(float) * (size_t)subs * BH + 255) & ~size_t(255));
}

template <int DK, bool GATED>
ret_status launch_state_dk(const void* k, const void* v, const float* decay, float* state_out, int B, int H, int N,
                           int dv, int subs, int sub_chunks, void* scratch, cudaStream_t st) {
    const int BH = B * H;
    // the state-only pass reads only K and V: the Q and O maps are placeholders over K and V
    CUtensorMap mk, mv;
    if (!make_map(&mk, k, DK, N, BH) || !make_map(&mv, v, dv, N, BH)) return RET_ERR_CUDA;
    uint8_t* sc = static_cast<uint8_t*>(scratch);
    float* states = subs > 1 ? reinterpret_cast<float*>(sc) : state_out;
    float* ldec = reinterpret_cast<float*>(sc + (subs > 1 ? sizeof(float) * (size_t)subs * BH * DK * dv : 0));
    Params prm{decay, nullptr, nullptr, states, ldec, H, N, dv, sub_chunks, 1, subs};
    auto k1 = state_tc_kernel<DK, GATED, false>;
    constexpr int smem1 = StateLayout<DK, state_tile(GATED)>::kSmemAlloc;
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1) != cudaSuccess)
        return RET_ERR_CUDA;
    if (launch_dependent(k1, dim3(dv / kDvS, BH, subs), kSThreads, smem1, st, mk, mv, prm) != cudaSuccess)
        return RET_ERR_CUDA;
    if (subs > 1) {
        if (launch_seg_prefix(nullptr, states, ldec, subs, BH, DK * dv, st) != cudaSuccess) return RET_ERR_CUDA;
        if (cudaMemcpyAsync(state_out, states + (size_t)(subs - 1) * BH * DK * dv, sizeof(float) * (size_t)BH * DK * dv,
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return RET_ERR_CUDA;
    }
    return RET_OK;
}

}  // namespace tc

// State-only tensor-core pass over a whole sequence; scratch from the stream-ordered allocator.
template <bool GATED>
ret_status tc_state_launch(const void* k, const void* v, const float* decay, float* state_out, int B, int H, int N,
                           int dk, int dv, cudaStream_t st) {
    int subs = 1, sub_chunks = 1;
    tc::state_plan(B, H, N, dv, subs, sub_chunks);
    void* scratch = nullptr;
    tc::keep_pool_memory();
    if (cudaMallocAsync(&scratch, tc::state_scratch_bytes(subs, B * H, dk, dv), st) != cudaSuccess) return RET_ERR_CUDA;
    ret_status r = RET_ERR_UNSUPPORTED;
    switch (dk) {
        case 64: r = tc::launch_state_dk<64, GATED>(k, v, decay, state_out, B, H, N, dv, subs, sub_chunks, scratch, st); break;
        case 128: r = tc::launch_state_dk<128, GATED>(k, v, decay, state_out, B, H, N, dv, subs, sub_chunks, scratch, st); break;
        case 256: r = tc::launch_state_dk<256, GATED>(k, v, decay, state_out, B, H, N, dv, subs, sub_chunks, scratch, st); break;
    }
    if (cudaFreeAsync(scratch, st) != cudaSuccess) return RET_ERR_CUDA;
    return r;
}

inline int tc_state_launches(int B, int H, int N, int dv) {
    int subs = 1, sub_chunks = 1;
    tc::state_plan(B, H, N, dv, subs, sub_chunks);
    return subs > 1 ? 2 : 1;  // state-only pass (+ prefix); the final copy is not a kernel
}

// Tensor-core path; a split sequence takes its scratch from the stream-ordered
// allocator and returns it on the same stream after the two launches.
template <bool GATED, bool REV = false>
ret_status tc_chunk_launch(const void* q, const void* k, const void* v, const float* decay, void* o,
                           const float* state_in, float* state_out, int B, int H, int N, int dk, int dv,
                           cudaStream_t st, int ldq = 0, int ldk = 0, int concurrent = 1, bool o_add = false) {
    const tc::Plan pl = tc::plan(B, H, N, dv, true, concurrent);
    void* scratch = nullptr;
    const size_t bytes = tc::scratch_bytes(pl, B * H, dk, dv, state_in != nullptr && state_in == state_out);
    if (bytes) tc::keep_pool_memory();
    if (bytes && cudaMallocAsync(&scratch, bytes, st) != cudaSuccess) return RET_ERR_CUDA;
    const ret_status r = tc::launch_with_scratch<GATED, REV>(q, k, v, decay, o, state_in, state_out, B, H, N, dk,
                                                             dv, pl, scratch, st, ldq, ldk, o_add);
    if (scratch && cudaFreeAsync(scratch, st) != cudaSuccess) return RET_ERR_CUDA;
    return r;
}

}  // namespace ret
