// Two-SM form of the tensor-core W4A8 product (steps 4-6 of "How it works" in
// the Keras guide "INT4 quantization in Keras"): a pair of CTAs in one
// cluster computes a 256-channel x 160-token tile with tcgen05.mma
// cta_group::2, each MMA spanning both SMs' tensor cores.
//
// Why a pair. Per SM and per 256 k, the one-SM kernel (gemm_tc.cuh) moves
// about 128 KB through shared memory (TMA writes of 48 KB of activations and
// 16 KB of packed weights, the unpack's 16 KB of reads, the MMAs' 48 KB of
// activation reads) against 768 tensor cycles of work: more than the
// 128 B/cycle shared memory gives, so it cannot keep the tensor pipe busy. In
// a pair each SM stages and serves only HALF of the token tile: the MMA reads
// B (the activations) from both SMs' shared memory at once.
//
// Data split of one MMA (M = 256, N = 160, K = 32, kind::i8):
//  * A (weights): rows 0-127 from the leader CTA's TMEM, 128-255 from the
//    peer's, same column address (each CTA widens its own 128 channels);
//  * B (activations): tokens 0-79 from the leader's shared memory, 80-159
//    from the peer's, same shared-memory address;
//  * D: rows 0-127 (the leader's channels) in the leader's TMEM, 128-255 in
//    the peer's, all 160 token columns.
// No TMA load is multicast: each CTA loads its own halves into its own shared
// memory. Only the leader (cluster rank 0) issues MMAs; the peer's widening and
// epilogue warps report to the leader's barriers with remote mbarrier arrives,
// and the MMA commits are multicast to both CTAs' barriers.
//
// Pipeline. One iteration is 256 k: 8 MMAs of 80 tensor cycles. (The issuing
// thread's wait per iteration costs about 200 tensor cycles that only a queue
// of several MMAs hides: a probe ran 4 MMAs plus one wait at 66 % of the
// pipe's rate and 8 MMAs plus one wait at 99 %.) Five shared-memory stages of
// 36 KB per CTA stage the loads, and three TMEM A slots of 64 columns (beside
// the two 160-column accumulators) let the widening of an iteration start
// while the MMAs of the two before it still run.
//
// Epilogue. Per 32-token chunk the four epilogue warps write their 128
// channels' results into a shared-memory staging tile, and one thread stores it
// with a TMA bulk tensor store (two staging buffers, so the math of one chunk
// overlaps the store of the previous). Individual 128-byte warp stores were
// measured to drain at only about 5 B/cycle per SM under the load traffic of
// the main loop. Where Y, its row stride or its row of N outputs is not
// 16-byte aligned the epilogue stores directly, as the one-SM kernel does.
//
// Warp roles per CTA: warp 0 TMA, warp 1 TMEM (and, in the leader, the MMA
// issue), warps 4-11 weight widening (two warpgroups), warps 12-15 epilogue.
// Every mbarrier wait is bounded; both CTAs meet at a cluster barrier before
// TMEM is released and before either exits, so no remote access outlives its
// target.
#pragma once

#include "gemm_tc.cuh"

namespace w4a8 {
namespace tcp {

using tc::BM;
using tc::MMA_K;
constexpr int BT = 160;               // tokens per pair tile (the MMA's N)
constexpr int HT = BT / 2;            // tokens staged per CTA
constexpr int PBK = 256;              // k per pipeline iteration
constexpr int XB = 128;               // k bytes per activation box (the 128-byte swizzle span)
constexpr int NBOX = PBK / XB;        // activation boxes per stage
constexpr int KSTEPS = PBK / MMA_K;   // MMAs per iteration
constexpr int STAGES = 5;
constexpr int A_SLOTS = 3;
constexpr int A_COLS = PBK / 4;       // TMEM columns per A slot
constexpr int W_ROW = PBK / 2;        // packed bytes per weight row and iteration
constexpr int ACT_BYTES = HT * PBK;   // NBOX 128B-swizzled boxes [HT][128 B]
constexpr int W_BYTES = BM * W_ROW;   // one 128B-swizzled box [BM][128 B]
constexpr int EPI_ROWS = 32;          // tokens per staged output chunk
constexpr int EPI_BYTES = EPI_ROWS * BM * 4;
constexpr int UNPACK_WG = 2;
constexpr int FIRST_UNPACK_WARP = 4;
constexpr int FIRST_EPI_WARP = FIRST_UNPACK_WARP + 4 * UNPACK_WG;
constexpr int NUM_THREADS = 32 * (FIRST_EPI_WARP + 4);
constexpr int TMEM_COLS = 512;
static_assert(2 * BT + A_SLOTS * A_COLS <= TMEM_COLS, "TMEM budget");
// The widening warps reuse A slot it % A_SLOTS once the stage barrier of
// iteration it - A_SLOTS has flipped; that barrier is not reused before
// iteration it - A_SLOTS + STAGES >= it, which cannot have been issued yet.
// (Which warpgroup widened the slot's previous iteration does not matter:
// the wait is on that iteration's MMAs.)
static_assert(STAGES >= A_SLOTS, "A-slot reuse waits on a stage barrier");
static_assert((HT * XB) % 1024 == 0 && W_BYTES % 1024 == 0, "swizzle atoms of whole boxes");
static_assert(W_ROW == 128, "weight tile rows span the 128-byte swizzle");

__host__ __device__ constexpr int d_col(int buf) { return buf * BT; }
__host__ __device__ constexpr int a_col(int slot) { return 2 * BT + slot * A_COLS; }

struct alignas(1024) Smem {
    uint8_t act[STAGES][ACT_BYTES];
    uint8_t wpk[STAGES][W_BYTES];
    uint8_t epi[2][EPI_BYTES];          // output staging: [32 tokens][128 channels]
    uint64_t full[STAGES];              // this CTA's TMA landed
    uint64_t empty[STAGES];             // MMAs reading the stage finished (multicast commit)
    uint64_t aready[A_SLOTS];           // leader: both CTAs' A slots written (8 warps)
    uint64_t acc_full[2];               // accumulator ready (multicast commit)
    uint64_t acc_empty[2];              // leader: both CTAs' epilogues drained (8 warps)
    uint64_t mma_done;                  // final drain (multicast commit)
    float rsx[BT];
    float tsx[BT];
    int32_t trs[BT];
    float tmin, tmax;                   // extreme sx of the epilogue's current tile
    uint32_t tmem_base;
    int abort;
};

// ---- pair forms of the tcgen05 wrappers ----
__device__ __forceinline__ void tmem_alloc2(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(ptx::smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_i8_ts2(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on the barrier at this shared-memory offset in both CTAs of the
// pair once every MMA this thread issued so far completed.
__device__ __forceinline__ void mma_commit2_both(uint64_t *bar) {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            ptx::smem_addr(bar)),
        "h"(mask)
        : "memory");
}
// Arrive on the leader's copy of a barrier (default release semantics, as
// for a local arrive). What the arrive publishes is the completion of this
// warp's tcgen05.st / tcgen05.ld, which tcgen05.wait and
// tcgen05.fence::before_thread_sync order before it; no generic-proxy data
// crosses the pair. (A release at cluster scope here was measured to cost
// about 1300 cycles per arrive on B200, which put it on the critical path of
// every pipeline iteration.)
__device__ __forceinline__ void mbar_arrive_leader(uint64_t *bar) {
    const uint32_t ra = ptx::mapa_shared(ptx::smem_addr(bar), 0u);
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(ra) : "memory");
}
// ---- TMA bulk tensor store of the output staging tile ----
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(ptx::smem_addr(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// At most one committed store group may still be reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Every committed store group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Epilogue of one 32-token chunk for one output channel into the staging
// tile (row j of the tile = token m0 + j, column = this thread's channel).
// The arithmetic is the one-SM kernel's (tc::epi_chunk): y = acc / (sx * sw)
// through the reciprocal product and one Markstein correction; EXACT takes
// the IEEE division instead (tiles whose scale products leave the range
// where the reciprocal form holds). Tokens past M are computed from the
// zero-filled rows and clipped by the store.
template <int FMT, bool BIAS, bool RELU, bool ZP, bool EXACT>
__device__ __forceinline__ void epi_stage(const uint32_t (&v)[32], uint8_t *stage, int col, float swn, float rswn,
                                          float bn, const float *__restrict__ tsx, const float *__restrict__ rsx,
                                          int32_t zpn, const int32_t *__restrict__ trs) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        int32_t acc = (int32_t)v[j] >> 4;  // the widened weights hold 16 q
        if constexpr (ZP) acc = (int32_t)((uint32_t)acc - (uint32_t)zpn * (uint32_t)trs[j]);
        if constexpr (FMT == tc::EPI_S32) {
            reinterpret_cast<int32_t *>(stage)[j * BM + col] = acc;
        } else {
            const float f = __int2float_rn(acc);
            float y;
            if constexpr (EXACT) {
                y = __fdiv_rn(f, __fmul_rn(tsx[j], swn));
            } else {
                const float d = __fmul_rn(tsx[j], swn);
                const float r = __fmul_rn(rsx[j], rswn);
                const float q0 = __fmul_rn(f, r);
                const float e = __fmaf_rn(-q0, d, f);
                y = __fmaf_rn(e, r, q0);
            }
            if constexpr (BIAS) y = __fadd_rn(y, bn);
            if constexpr (RELU) y = y > 0.0f ? y : 0.0f;
            if constexpr (FMT == tc::EPI_BF16)
                reinterpret_cast<__nv_bfloat16 *>(stage)[j * BM + col] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float *>(stage)[j * BM + col] = y;
        }
    }
}

template <int FMT, bool BIAS, bool RELU, bool ZP>
__device__ __forceinline__ void epi_stage_any(bool exact, const uint32_t (&v)[32], uint8_t *stage, int col,
                                              float swn, float rswn, float bn, const float *__restrict__ tsx,
                                              const float *__restrict__ rsx, int32_t zpn,
                                              const int32_t *__restrict__ trs) {
    if (FMT != tc::EPI_S32 && exact)
        epi_stage<FMT, BIAS, RELU, ZP, true>(v, stage, col, swn, rswn, bn, tsx, rsx, zpn, trs);
    else
        epi_stage<FMT, BIAS, RELU, ZP, false>(v, stage, col, swn, rswn, bn, tsx, rsx, zpn, trs);
}

// UNPACK: tc::UNPACK_X16 (natural k order) or tc::UNPACK_X16_PERM (the
// activation pass's k-permuted order). K <= tc::TC_X16_MAX_K.
// tma_out: tm_y describes Y and the epilogue stores through staging tiles.
template <int UNPACK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_gemm_tc_pair(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
               const __grid_constant__ CUtensorMap tm_y, int tma_out, int M, int N, int K,
               const float *__restrict__ sx, const float *__restrict__ sw, const float *__restrict__ bias,
               unsigned flags, void *__restrict__ Y, int ldy, ZpArgs zpa) {
    static_assert(UNPACK == tc::UNPACK_X16 || UNPACK == tc::UNPACK_X16_PERM, "16 q forms");
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
    const int num_kb = (K + PBK - 1) / PBK;
    const int tiles_m = (M + BT - 1) / BT;
    const int tiles_n = (N + 2 * BM - 1) / (2 * BM);
    const int num_tiles = tiles_m * tiles_n;
    const int my_tiles = (num_tiles - pair + npairs - 1) / npairs;
    const int total = my_tiles * num_kb;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < A_SLOTS; ++a) ptx::mbar_init(&sm.aready[a], 8);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&sm.acc_full[b], 1);
            ptx::mbar_init(&sm.acc_empty[b], 8);
        }
        ptx::mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_w);
        ptx::prefetch_tensormap(&tm_x);
        if (tma_out) ptx::prefetch_tensormap(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc2(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish2();
    }
    ptx::tc_fence_before();
    // both CTAs' barriers initialized and TMEM allocated before any remote use
    ptx::cluster_arrive_release();
    ptx::cluster_wait_acquire();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // With W4A8_STATIC_WEIGHTS the first stages' weight tiles are requested
    // before the dependency wait (the stages are all free at the start); the
    // activations are read only after it.
    auto load_weights = [&](int stage, int n_tile, int kb) {
        ptx::mbar_arrive_expect_tx(&sm.full[stage], ACT_BYTES + W_BYTES);
        ptx::tma_load_2d(sm.wpk[stage], &tm_w, kb * W_ROW, n_tile * 2 * BM + (int)rank * BM, &sm.full[stage]);
    };
    const int pre_w = (flags & W4A8_STATIC_WEIGHTS) ? min(STAGES, total) : 0;
    if (warp == 0 && lane == 0)
        for (int it = 0; it < pre_w; ++it) load_weights(it, (pair + (it / num_kb) * npairs) / tiles_m, it % num_kb);
    __syncwarp();

    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer (each CTA: its halves)
        if (lane == 0) {
            int stage = 0, it = 0;
            uint32_t phase = 0, issued = 0, last_par = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                const int n_tile = tile / tiles_m, m_tile = tile % tiles_m;
                const int m0 = m_tile * BT + (int)rank * HT;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    if (it >= pre_w) {
                        if (!ptx::mbar_wait(&sm.empty[stage], phase ^ 1, abort)) { ok = false; break; }
                        load_weights(stage, n_tile, kb);
                    }
#pragma unroll
                    for (int h = 0; h < NBOX; ++h)
                        ptx::tma_load_2d(sm.act[stage] + h * HT * XB, &tm_x, kb * PBK + h * XB, m0, &sm.full[stage]);
                    issued |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            // Drain: every load this thread issued lands before the CTA exits.
            if (!ok)
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s)) ptx::mbar_wait_drain(&sm.full[s], (last_par >> s) & 1u);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer (leader only)
        // The widening warps of both CTAs arrive on aready only after their
        // own wait on full[] of the same iteration, so once aready flipped
        // both CTAs' activation halves have landed as well.
        if (leader && lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_i8(2 * BM, BT);
            int stage = 0, slot = 0, kb = 0, buf = 0;
            uint32_t aphase = 0, bphase = 0;
            bool ok = total > 0 ? ptx::mbar_wait(&sm.aready[0], 0, abort) : true;
            for (int it = 0; it < total && ok; ++it) {
                if (kb == 0 && !ptx::mbar_wait(&sm.acc_empty[buf], bphase ^ 1u, abort)) break;
                ptx::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)d_col(buf);
                const uint32_t a = tmem + (uint32_t)a_col(slot);
                const uint32_t b = ptx::smem_addr(sm.act[stage]);
                // k step kk reads activation box kk / 4 at byte offset 32 (kk % 4)
                constexpr int KPB = XB / MMA_K;
#pragma unroll
                for (int kk = 0; kk < KSTEPS - 1; ++kk)
                    mma_i8_ts2(d, a + kk * (MMA_K / 4), ptx::sdesc_k_sw128(b + (kk / KPB) * HT * XB + (kk % KPB) * MMA_K),
                               idesc, (kb | kk) != 0);
                int nstage = stage + 1, nslot = slot + 1;
                uint32_t naphase = aphase;
                if (nstage == STAGES) nstage = 0;
                if (nslot == A_SLOTS) { nslot = 0; naphase ^= 1u; }
                // wait for the next operands while the queued MMAs run
                const bool next_ok = it + 1 < total ? ptx::mbar_wait(&sm.aready[nslot], naphase, abort) : true;
                mma_i8_ts2(d, a + (KSTEPS - 1) * (MMA_K / 4),
                           ptx::sdesc_k_sw128(b + ((KSTEPS - 1) / KPB) * HT * XB + ((KSTEPS - 1) % KPB) * MMA_K), idesc,
                           1u);
                mma_commit2_both(&sm.empty[stage]);
                if (++kb == num_kb) {
                    mma_commit2_both(&sm.acc_full[buf]);
                    kb = 0;
                    if (++buf == 2) { buf = 0; bphase ^= 1u; }
                }
                stage = nstage;
                slot = nslot;
                aphase = naphase;
                ok = next_ok;
            }
            // Both CTAs' mma_done flip once every MMA issued above has
            // finished (at once when none was issued).
            if (total > 0) mma_commit2_both(&sm.mma_done);
        }
    } else if (warp >= FIRST_UNPACK_WARP && warp < FIRST_EPI_WARP) {
        // ---------------------------------------------------- weight widening (each CTA: its 128 rows)
        // Thread r owns channel row r of this CTA's half: 128 packed bytes per
        // iteration, read from the 128B-swizzled tile (16-byte chunk c of row
        // r sits at chunk c ^ (r & 7)), widened to 256 INT8 and stored to
        // TMEM lane r, 64 columns (two stores of 32).
        const int q = warp & 3;
        const int wg = (warp - FIRST_UNPACK_WARP) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int swz = r & 7;
        bool ok = true;
        for (int it = wg; it < total && ok; it += UNPACK_WG) {
            const int stage = it % STAGES;
            const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
            const int slot = it % A_SLOTS;
            // the slot was last read by iteration it - A_SLOTS, whose MMAs
            // completed when that iteration's stage barrier flipped
            bool got = ptx::mbar_wait(&sm.full[stage], phase, abort);
            if (got && it >= A_SLOTS) {
                const int j = it - A_SLOTS;
                got = ptx::mbar_wait(&sm.empty[j % STAGES], (uint32_t)(j / STAGES) & 1u, abort);
            }
            ok = __all_sync(0xffffffffu, got);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint8_t *row = sm.wpk[stage] + r * W_ROW;
#pragma unroll
            for (int half = 0; half < W_ROW / 64; ++half) {
                uint32_t out[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + 16 * ((4 * half + c) ^ swz));
                    const uint32_t p[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t lo = (p[j] << 4) & 0xF0F0F0F0u;  // 16 q of k0 k2 k4 k6
                        const uint32_t hi = p[j] & 0xF0F0F0F0u;         // 16 q of k1 k3 k5 k7
                        if constexpr (UNPACK == tc::UNPACK_X16_PERM) {
                            out[8 * c + 2 * j] = lo;
                            out[8 * c + 2 * j + 1] = hi;
                        } else {
                            out[8 * c + 2 * j] = __byte_perm(lo, hi, 0x5140);      // k0 k1 k2 k3
                            out[8 * c + 2 * j + 1] = __byte_perm(lo, hi, 0x7362);  // k4 k5 k6 k7
                        }
                    }
                }
                ptx::tmem_st_32x32b_x32(tmem + lane_base + (uint32_t)(a_col(slot) + 32 * half), out);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_leader(&sm.aready[slot]);
        }
    } else if (warp >= FIRST_EPI_WARP) {
        // ---------------------------------------------------- epilogue (each CTA: its 128 channels)
        const int q = warp & 3;
        const int et = threadIdx.x - 32 * FIRST_EPI_WARP;  // 0..127: this CTA's channel column
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int buf = 0, sb = 0;
        uint32_t acc_phase = 0;
        const unsigned fmt = flags & W4A8_OUT_MASK;
        const int epi_mode = fmt == W4A8_OUT_S32 ? 8
                             : (fmt == W4A8_OUT_BF16 ? 4 : 0) + (bias ? 2 : 0) + ((flags & W4A8_RELU) ? 1 : 0);
        const bool zp = zpa.zp != nullptr;
        for (int tile = pair; tile < num_tiles; tile += npairs) {
            const int n_tile = tile / tiles_m, m_tile = tile % tiles_m;
            const int m_base = m_tile * BT;
            const int n_base = n_tile * 2 * BM + (int)rank * BM;
            // scales of this tile's tokens (the previous tile's readers are
            // past the named barrier at its end)
            for (int c = et; c < BT; c += 128) {
                const int m = m_base + c;
                const float v = m < M ? ld_dep(sx + m) : 1.0f;
                sm.tsx[c] = v;
                sm.rsx[c] = __frcp_rn(v);
                sm.trs[c] = (zp && m < M) ? ld_dep_s32(zpa.rowsum + m) : 0;
            }
            ptx::bar_sync(1, 128);
            if (warp == FIRST_EPI_WARP) {
                // extremes of the tile's sx (all positive or zero): whether every
                // product sx * sw of a channel lies where the reciprocal form holds
                float lo = 3.4e38f, hi = 0.0f;
                for (int c = lane; c < BT; c += 32) {
                    lo = fminf(lo, sm.tsx[c]);
                    hi = fmaxf(hi, sm.tsx[c]);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
                }
                if (lane == 0) {
                    sm.tmin = lo;
                    sm.tmax = hi;
                }
            }
            // One decision for all four epilogue warps (this barrier also
            // publishes the tile's tables): a warp that gave up must not leave
            // the others waiting at a named barrier.
            if (!ptx::bar_and(1, 128, ptx::mbar_wait(&sm.acc_full[buf], acc_phase, abort))) break;
            ptx::tc_fence_after();
            const int n = n_base + et;
            const bool n_ok = n < N;
            const float swn = n_ok ? ld_dep(sw + n) : 1.0f;
            const float rswn = __frcp_rn(swn);
            const float bn = (bias && n_ok) ? ld_dep(bias + n) : 0.0f;
            const int32_t zpn = (zp && n_ok) ? ld_dep_s32(zpa.zp + n) - 8 : 0;
            const float dlo = __fmul_rn(sm.tmin, swn), dhi = __fmul_rn(sm.tmax, swn);
            const bool exact = !(dlo >= 0x1p-94f && dhi <= 0x1p126f);
#pragma unroll 1
            for (int c0 = 0; c0 < BT; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem + lane_base + (uint32_t)(d_col(buf) + c0), v);
                ptx::tmem_wait_ld();
                const int mrem = M - (m_base + c0);
                if (mrem <= 0) break;
                const int m0 = m_base + c0;
                const float *tsx = sm.tsx + c0, *rsx = sm.rsx + c0;
                const int32_t *trs = sm.trs + c0;
                if (tma_out) {
                    // staging buffer sb: the store issued from it two chunks ago
                    // has finished reading it once at most one group is pending
                    if (et == 0) bulk_wait_read_1();
                    ptx::bar_sync(1, 128);
                    uint8_t *stg = sm.epi[sb];
#define W4A8_EPS(F, B, R)                                                                                   \
    (zp ? epi_stage_any<F, B, R, true>(exact, v, stg, et, swn, rswn, bn, tsx, rsx, zpn, trs)              \
        : epi_stage_any<F, B, R, false>(exact, v, stg, et, swn, rswn, bn, tsx, rsx, zpn, trs))
                    switch (epi_mode) {
                        case 0: W4A8_EPS(tc::EPI_F32, false, false); break;
                        case 1: W4A8_EPS(tc::EPI_F32, false, true); break;
                        case 2: W4A8_EPS(tc::EPI_F32, true, false); break;
                        case 3: W4A8_EPS(tc::EPI_F32, true, true); break;
                        case 4: W4A8_EPS(tc::EPI_BF16, false, false); break;
                        case 5: W4A8_EPS(tc::EPI_BF16, false, true); break;
                        case 6: W4A8_EPS(tc::EPI_BF16, true, false); break;
                        case 7: W4A8_EPS(tc::EPI_BF16, true, true); break;
                        default: W4A8_EPS(tc::EPI_S32, false, false); break;
                    }
#undef W4A8_EPS
                    fence_proxy_async_smem();  // the staging writes, before the async-proxy store reads them
                    ptx::bar_sync(1, 128);
                    if (et == 0 && n_base < N) {
                        tma_store_2d(&tm_y, stg, n_base, m0);
                        bulk_commit_group();
                    }
                    sb ^= 1;
                } else {
#define W4A8_EPI2(F, B, R) \
    tc::epi_chunk_any<F, B, R, 4>(v, Y, ldy, m0, mrem, n, n_ok, swn, rswn, bn, tsx, rsx, zpn, trs)
                    switch (epi_mode) {
                        case 0: W4A8_EPI2(tc::EPI_F32, false, false); break;
                        case 1: W4A8_EPI2(tc::EPI_F32, false, true); break;
                        case 2: W4A8_EPI2(tc::EPI_F32, true, false); break;
                        case 3: W4A8_EPI2(tc::EPI_F32, true, true); break;
                        case 4: W4A8_EPI2(tc::EPI_BF16, false, false); break;
                        case 5: W4A8_EPI2(tc::EPI_BF16, false, true); break;
                        case 6: W4A8_EPI2(tc::EPI_BF16, true, false); break;
                        case 7: W4A8_EPI2(tc::EPI_BF16, true, true); break;
                        default: W4A8_EPI2(tc::EPI_S32, false, false); break;
                    }
#undef W4A8_EPI2
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_leader(&sm.acc_empty[buf]);
            if (++buf == 2) { buf = 0; acc_phase ^= 1; }
            ptx::bar_sync(1, 128);  // the tables are rewritten next tile
        }
        // the output stores have completed before the CTA exits
        if (et == 0 && tma_out) bulk_wait_all();
    }

    // Every MMA of the pair has finished before TMEM is released: the leader's
    // final commit reaches both CTAs' mma_done.
    if (warp == 1) {
        if (total > 0 && lane == 0) ptx::mbar_wait_drain(&sm.mma_done, 0);
        __syncwarp();
    }
    ptx::tc_fence_before();
    __syncthreads();
    // the pair meets before TMEM is released and before either CTA exits
    ptx::cluster_arrive_release();
    ptx::cluster_wait_acquire();
    ptx::tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc2(tmem, TMEM_COLS);
    }
}

inline size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Clusters of two that the device holds at once (queried once per process
// for the first device that asks; the pool's devices are alike).
template <int UNPACK>
inline int resident_pairs(const cudaLaunchConfig_t &cfg_in, int sm_count) {
    static std::once_flag once;
    static int n = 0;
    std::call_once(once, [&] {
        cudaLaunchConfig_t cfg = cfg_in;
        cfg.gridDim = dim3((unsigned)(sm_count & ~1));
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, k_gemm_tc_pair<UNPACK>, &cfg) == cudaSuccess) n = c;
        else (void)cudaGetLastError();
    });
    return n < sm_count / 2 ? n : sm_count / 2;
}

template <int UNPACK>
inline w4a8_status launch(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                          const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy, int sm_count,
                          cudaStream_t stream, ZpArgs zpa) {
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(k_gemm_tc_pair<UNPACK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem_bytes());
    });
    if (attr_err != cudaSuccess) return W4A8_ERR_CUDA;
    CUtensorMap tm_w, tm_x, tm_y;
    if (!tc::make_map_u8(&tm_w, Wp, (uint64_t)ldp, (uint64_t)N, (uint64_t)ldp, W_ROW, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tc::make_map_u8(&tm_x, Xq, (uint64_t)ldq, (uint64_t)M, (uint64_t)ldq, XB, HT, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    // The staged epilogue stores through a tensor map of Y, which needs a
    // 16-byte aligned base and row stride, and a row of N outputs that ends
    // on a 16-byte boundary: the store's bounds check on the inner dimension
    // was observed to work in 16-byte units on B200 (a box clipped at
    // N = 270 f32 outputs also wrote outputs 270 and 271). Otherwise the
    // epilogue stores directly.
    const unsigned fmt = flags & W4A8_OUT_MASK;
    const size_t esz = fmt == W4A8_OUT_BF16 ? 2 : 4;
    const CUtensorMapDataType yt = fmt == W4A8_OUT_BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : fmt == W4A8_OUT_S32 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    int tma_out = 0;
    memset(&tm_y, 0, sizeof(tm_y));
    if ((reinterpret_cast<uintptr_t>(Y) & 15) == 0 && ((size_t)ldy * esz) % 16 == 0 && ((size_t)N * esz) % 16 == 0 &&
        M > 0)
        tma_out = tc::make_map_2d(&tm_y, yt, Y, (uint64_t)N, (uint64_t)M, (uint64_t)ldy * esz, BM, EPI_ROWS,
                                  CU_TENSOR_MAP_SWIZZLE_NONE)
                      ? 1
                      : 0;
    const long long tiles = (long long)((M + BT - 1) / BT) * ((N + 2 * BM - 1) / (2 * BM));
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // one persistent pair per pair of SMs that can hold one at a time
    const int resident = resident_pairs<UNPACK>(cfg, sm_count);
    if (resident < 1) return W4A8_ERR_UNSUPPORTED;
    const long long pairs = tiles < resident ? tiles : resident;
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_gemm_tc_pair<UNPACK>, tm_w, tm_x, tm_y, tma_out, M, N, K, sx, sw,
                                       bias, flags, Y, ldy, zpa);
    return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

}  // namespace tcp
}  // namespace w4a8
