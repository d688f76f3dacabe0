// Tensor-core path of the quantized product on sm_100a (steps 4-6 of "How it
// works" in the Keras guide "INT4 quantization in Keras"): packed INT4 weights
// are unpacked to INT8 on chip and multiplied with INT8 activations by
// tcgen05.mma kind::i8, accumulating in INT32 in tensor memory (TMEM); the
// epilogue dequantizes acc / (sx * sw) and applies bias and ReLU.
//
// The product is computed transposed, D^T[n][m] = sum_k q[n][k] * xq[m][k]:
//  * A (M_mma = 128 output channels x K) comes from TMEM. A warpgroup reads the
//    packed tile that TMA put in shared memory, sign-extends the nibbles in
//    registers and writes the INT8 rows into TMEM with tcgen05.st, so the
//    unpacked weights never travel through shared memory.
//  * B (N_mma = BT tokens x K) is the INT8 activation tile, loaded by TMA with
//    128-byte swizzling and read by the MMA through a shared-memory descriptor.
//  * D lives in TMEM with output channels on lanes and tokens on columns, so
//    an epilogue thread owns one output channel (one weight scale, one bias)
//    and a warp stores 32 consecutive channels of a token row at once.
//
// One persistent CTA per SM walks the (channel tile, token tile) grid.
// Warp roles: warp 0 issues TMA loads, warp 1 owns TMEM and issues the MMAs,
// warps 4-11 (two warpgroups) unpack weights, warps 12-15 run the epilogue.
// Shared-memory stages and TMEM A slots form rings; the
// accumulator is double-buffered so the epilogue of one tile overlaps the
// main loop of the next. Every mbarrier wait is bounded (see ptx::mbar_wait).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace tc {

constexpr int BM = 128;            // output channels per tile (MMA M)
constexpr int BK = 256;            // k per stage (one pipeline iteration)
constexpr int MMA_K = 32;          // k per kind::i8 instruction
constexpr int XBOX = 128;          // bytes of k per activation TMA box (the 128-byte swizzle span)
// The tensor core queues about one MMA ahead of the issuing thread, so every
// stretch of other work on that thread (barrier waits, the commit, loop
// bookkeeping) longer than one MMA leaves the pipe idle. Hence wide MMAs (a
// token tile of BT = 192 gives N = 192, 96 tensor cycles each) and 8 of them
// per pipeline iteration (BK = 256). Smaller token tiles (128, 64) serve
// layers whose few rows or few tiles would leave a 192-token grid padded or
// mostly idle; the host picks BT per call.
//
// Two rings per token tile. Shared-memory stages (TMA -> unpack/MMA) take
// 192 KB, which also keeps a second CTA (that would block in tcgen05.alloc
// of the whole TMEM) off the SM. TMEM A slots (unpack -> MMA) of 64 columns
// sit next to the two BT-column accumulators.
template <int BT> struct Ring;
template <> struct Ring<192> { static constexpr int STAGES = 3, A_SLOTS = 2; };  // 3 x 64 KB, 384 + 128 cols
template <> struct Ring<128> { static constexpr int STAGES = 4, A_SLOTS = 4; };  // 4 x 48 KB, 256 + 256 cols
template <> struct Ring<64> { static constexpr int STAGES = 6, A_SLOTS = 4; };   // 6 x 32 KB, 128 + 256 cols
// The W8A8 form: weight tiles of one byte per code are twice as large, so
// fewer stages fit the same shared memory. A 192-token tile would keep only
// 2 stages of 80 KB; measured on B200 that ring was too shallow (1194 TOPS at
// M = 2048, K = 4096, N = 11008 against 1847 with 160 tokens and 3 stages),
// so W8A8 runs BT = 160, 128 or 64.
template <int BT> struct Ring8;
template <> struct Ring8<160> { static constexpr int STAGES = 3, A_SLOTS = 2; };  // 3 x 72 KB, 320 + 128 cols
template <> struct Ring8<128> { static constexpr int STAGES = 3, A_SLOTS = 2; };  // 3 x 64 KB, 256 + 128 cols
template <> struct Ring8<64> { static constexpr int STAGES = 4, A_SLOTS = 4; };   // 4 x 48 KB, 128 + 256 cols
// Unpack warpgroups: pipeline iteration `it` is unpacked by warpgroup
// it % UNPACK_WG, so the groups overlap their shared-memory reads, integer
// work and TMEM stores.
constexpr int UNPACK_WG = 2;
static_assert(BK % XBOX == 0 && XBOX % MMA_K == 0, "activation boxes hold whole MMA k steps");
constexpr int FIRST_UNPACK_WARP = 4;
constexpr int FIRST_EPI_WARP = FIRST_UNPACK_WARP + 4 * UNPACK_WG;
constexpr int NUM_THREADS = 32 * (FIRST_EPI_WARP + 4);
constexpr int TMEM_COLS = 512;
constexpr int A_COLS = BK / 4;     // TMEM columns per A slot (4 INT8 per column)

// How the weight warpgroups widen nibbles to the INT8 A operand.
//  UNPACK_SEXT: sign-extend each nibble (byte = q), then restore k order with
//      two byte permutes. Any K.
//  UNPACK_X16:  keep each nibble in the high half of its byte, so the byte is
//      exactly 16*q as INT8 (q in [-8, 7] gives 16q in [-128, 112]); the
//      accumulator is then exactly 16*acc and the epilogue shifts it back.
//      Two masks and one shift per 8 codes, plus the two byte permutes.
//      Each term 16 q * xq is at most 128 * 127 in size, so this needs
//      128 * 127 * K < 2^31, i.e. K <= TC_X16_MAX_K.
//  UNPACK_X16_PERM: as UNPACK_X16 without the byte permutes: the activations
//      were stored with each group of 8 k reordered to k0 k2 k4 k6 k1 k3 k5 k7
//      (see k_act_quant), which is the order the masks produce.
//  UNPACK_NONE: the W8A8 path - the weight tile already holds one INT8 code
//      per byte (two 128-byte boxes per row and stage, like the
//      activations), and the weight warps copy it into TMEM unchanged.
enum { UNPACK_SEXT = 0, UNPACK_X16 = 1, UNPACK_X16_PERM = 2, UNPACK_NONE = 3 };
constexpr int TC_X16_MAX_K = 131072;

// Ring sizes and the weight tile of a kernel form.
template <int BT, int UNPACK>
struct Cfg {
    static constexpr bool W8 = UNPACK == UNPACK_NONE;
    using R = std::conditional_t<W8, Ring8<BT>, Ring<BT>>;
    static constexpr int STAGES = R::STAGES;
    static constexpr int A_SLOTS = R::A_SLOTS;
    static constexpr int W_TILE_BYTES = W8 ? BM * BK : BM * BK / 2;
    static constexpr int SHIFT = (UNPACK == UNPACK_X16 || UNPACK == UNPACK_X16_PERM) ? 4 : 0;
};

template <int BT, int UNPACK>
struct alignas(1024) Smem {
    using C = Cfg<BT, UNPACK>;
    uint8_t act[C::STAGES][BT * BK];          // activation tiles: BK / XBOX boxes of [BT][128 B], 128B-swizzled
    uint8_t wpk[C::STAGES][C::W_TILE_BYTES];  // weight tiles: [BM][128 B] packed, or W8: two boxes of [BM][128 B]
    uint64_t full[C::STAGES];                 // TMA landed (tx-count barrier)
    uint64_t empty[C::STAGES];                // MMAs reading the stage finished
    uint64_t aready[C::A_SLOTS];              // A slot written to TMEM (4 unpack warps)
    uint64_t acc_full[2];                // accumulator ready for the epilogue
    uint64_t acc_empty[2];               // epilogue drained the accumulator (4 warps)
    uint64_t mma_done;                   // final drain of the MMA pipe
    float rsx[BT];                       // 1/sx of the epilogue's current token tile
    float tsx[BT];                       // sx of the same tokens
    int32_t trs[BT];                     // row sums of the same tokens (zero-point form; else 0)
    uint32_t tmem_base;
    int abort;
};

template <int BT>
constexpr int d_col(int buf) { return buf * BT; }
template <int BT>
constexpr int a_col(int slot) { return 2 * BT + slot * A_COLS; }

// Epilogue of one 32-token chunk for one output channel (this thread's TMEM
// lane): dequantize, bias, ReLU, store. Every choice is a template argument so
// the unrolled loop holds no branches (runtime branches per element made this
// loop several times slower); a chunk cut by the end of M takes the predicated
// form. v = raw TMEM words, SHIFT = 4 when they hold 16*acc.
enum { EPI_F32 = 0, EPI_BF16 = 1, EPI_S32 = 2 };

// Returns true when some d = sx * sw of the chunk lies outside 2^-94..2^126,
// where the reciprocal form is not valid (its correction needs a normal 1/d
// and a finite f * r for |f| < 2^31); the caller then redoes the chunk with
// the IEEE division (epi_chunk_exact), which keeps the rare path out of this
// unrolled loop.
template <int FMT, bool BIAS, bool RELU, int SHIFT, bool FULL>
__device__ __forceinline__ bool epi_chunk(const uint32_t (&v)[32], void *__restrict__ Y, int ldy, int m0, int mrem,
                                          int n, bool n_ok, float swn, float rswn, float bn,
                                          const float *__restrict__ tsx, const float *__restrict__ rsx,
                                          int32_t zpn, const int32_t *__restrict__ trs) {
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (!FULL && j >= mrem) break;
        // zero-point correction in modular INT32 arithmetic: exact whenever
        // the corrected accumulator fits INT32, as the method's does
        const int32_t acc = (int32_t)((uint32_t)((int32_t)v[j] >> SHIFT) - (uint32_t)zpn * (uint32_t)trs[j]);
        const size_t off = (size_t)(m0 + j) * (size_t)ldy + (size_t)n;
        if constexpr (FMT == EPI_S32) {
            if (n_ok) static_cast<int32_t *>(Y)[off] = acc;
        } else {
            const float f = __int2float_rn(acc);
            const float d = __fmul_rn(tsx[j], swn);
            const float r = __fmul_rn(rsx[j], rswn);
            const float q0 = __fmul_rn(f, r);
            const float e = __fmaf_rn(-q0, d, f);
            float y = __fmaf_rn(e, r, q0);
            bad |= !(d >= 0x1p-94f && d <= 0x1p126f);
            if constexpr (BIAS) y = __fadd_rn(y, bn);
            if constexpr (RELU) y = y > 0.0f ? y : 0.0f;
            if constexpr (FMT == EPI_BF16) {
                if (n_ok) static_cast<__nv_bfloat16 *>(Y)[off] = __float2bfloat16_rn(y);
            } else {
                if (n_ok) static_cast<float *>(Y)[off] = y;
            }
        }
    }
    return bad;
}

// The same chunk with y = float(acc) / (sx * sw) by IEEE division (extreme
// scale products only).
template <int FMT, bool BIAS, bool RELU, int SHIFT>
__device__ __noinline__ void epi_chunk_exact(const uint32_t (&v)[32], void *__restrict__ Y, int ldy, int m0,
                                             int mrem, int n, bool n_ok, float swn, float bn,
                                             const float *__restrict__ tsx, int32_t zpn,
                                             const int32_t *__restrict__ trs) {
#pragma unroll 1
    for (int j = 0; j < 32 && j < mrem; ++j) {
        const int32_t acc = (int32_t)((uint32_t)((int32_t)v[j] >> SHIFT) - (uint32_t)zpn * (uint32_t)trs[j]);
        const float y0 = __fdiv_rn(__int2float_rn(acc), __fmul_rn(tsx[j], swn));
        float y = y0;
        if constexpr (BIAS) y = __fadd_rn(y, bn);
        if constexpr (RELU) y = y > 0.0f ? y : 0.0f;
        const size_t off = (size_t)(m0 + j) * (size_t)ldy + (size_t)n;
        if constexpr (FMT == EPI_BF16) {
            if (n_ok) static_cast<__nv_bfloat16 *>(Y)[off] = __float2bfloat16_rn(y);
        } else {
            if (n_ok) static_cast<float *>(Y)[off] = y;
        }
    }
}

template <int FMT, bool BIAS, bool RELU, int SHIFT>
__device__ __forceinline__ void epi_chunk_any(const uint32_t (&v)[32], void *__restrict__ Y, int ldy, int m0,
                                              int mrem, int n, bool n_ok, float swn, float rswn, float bn,
                                              const float *__restrict__ tsx, const float *__restrict__ rsx,
                                              int32_t zpn, const int32_t *__restrict__ trs) {
    const bool bad = mrem >= 32 ? epi_chunk<FMT, BIAS, RELU, SHIFT, true>(v, Y, ldy, m0, mrem, n, n_ok, swn, rswn, bn,
                                                                          tsx, rsx, zpn, trs)
                                : epi_chunk<FMT, BIAS, RELU, SHIFT, false>(v, Y, ldy, m0, mrem, n, n_ok, swn, rswn,
                                                                           bn, tsx, rsx, zpn, trs);
    if constexpr (FMT != EPI_S32) {
        if (bad) epi_chunk_exact<FMT, BIAS, RELU, SHIFT>(v, Y, ldy, m0, mrem, n, n_ok, swn, bn, tsx, zpn, trs);
    }
}

template <int BT, int UNPACK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
          int M, int N, int K, const float *__restrict__ sx, const float *__restrict__ sw,
          const float *__restrict__ bias, unsigned flags, void *__restrict__ Y, int ldy, ZpArgs zpa) {
    constexpr int STAGES = Cfg<BT, UNPACK>::STAGES;
    constexpr int A_SLOTS = Cfg<BT, UNPACK>::A_SLOTS;
    constexpr int W_TILE_BYTES = Cfg<BT, UNPACK>::W_TILE_BYTES;
    static_assert(A_SLOTS % UNPACK_WG == 0, "each warpgroup owns fixed TMEM slots");
    // The unpack warps reuse A slot it % A_SLOTS once the stage barrier of
    // iteration it - A_SLOTS has flipped; that barrier is not reused before
    // iteration it - A_SLOTS + STAGES >= it, which cannot have run yet.
    static_assert(STAGES >= A_SLOTS, "A-slot reuse waits on a stage barrier");
    static_assert(2 * BT + A_SLOTS * A_COLS <= TMEM_COLS, "TMEM budget");
    static_assert(BT % 32 == 0 && BT >= 32 && BT <= 256, "token tile");
    extern __shared__ uint8_t smem_raw[];
    Smem<BT, UNPACK> &sm = *reinterpret_cast<Smem<BT, UNPACK> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_kb = (K + BK - 1) / BK;
    const int tiles_m = (M + BT - 1) / BT;
    const int tiles_n = (N + BM - 1) / BM;
    const int num_tiles = tiles_m * tiles_n;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < A_SLOTS; ++a) ptx::mbar_init(&sm.aready[a], 4);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&sm.acc_full[b], 1);
            ptx::mbar_init(&sm.acc_empty[b], 4);
        }
        ptx::mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_w);
        ptx::prefetch_tensormap(&tm_x);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&sm.tmem_base, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // Weight tiles of one pipeline iteration into a stage (the stage's full
    // barrier then also waits for the activation tile).
    auto load_weights = [&](int stage, int n_tile, int kb) {
        ptx::mbar_arrive_expect_tx(&sm.full[stage], BT * BK + W_TILE_BYTES);
        if constexpr (Cfg<BT, UNPACK>::W8) {
#pragma unroll
            for (int h = 0; h < BK / XBOX; ++h)
                ptx::tma_load_2d(sm.wpk[stage] + h * BM * XBOX, &tm_w, kb * BK + h * XBOX, n_tile * BM,
                                 &sm.full[stage]);
        } else {
            ptx::tma_load_2d(sm.wpk[stage], &tm_w, kb * (BK / 2), n_tile * BM, &sm.full[stage]);
        }
    };
    // With W4A8_STATIC_WEIGHTS the weights are final at launch: the first
    // stages' weight tiles are requested before the dependency wait (the
    // stages are all free at the start), so they overlap the previous
    // kernel's tail. The activations are read only after the wait.
    const int my_iters = ((num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * num_kb;
    const int pre_w = (flags & W4A8_STATIC_WEIGHTS) ? min(STAGES, my_iters) : 0;
    if (warp == 0 && lane == 0) {
        for (int it = 0; it < pre_w; ++it)
            load_weights(it, ((int)blockIdx.x + (it / num_kb) * (int)gridDim.x) / tiles_m, it % num_kb);
    }
    __syncwarp();

    // Dependents may launch once every CTA of this grid is resident; the
    // activations and scales come from the previous kernel, so wait for it.
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;  // bit s: stage s has a load whose landing we have not seen
            uint32_t last_par = 0;
            bool ok = true;
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int n_tile = tile / tiles_m, m_tile = tile % tiles_m;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    if (it >= pre_w) {
                        if (!ptx::mbar_wait(&sm.empty[stage], phase ^ 1, abort)) { ok = false; break; }
                        load_weights(stage, n_tile, kb);
                    }
#pragma unroll
                    for (int h = 0; h < BK / XBOX; ++h)
                        ptx::tma_load_2d(sm.act[stage] + h * BT * XBOX, &tm_x, kb * BK + h * XBOX, m_tile * BT,
                                         &sm.full[stage]);
                    issued |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // Drain: every load this thread issued lands before the CTA exits.
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s)) ptx::mbar_wait_drain(&sm.full[s], (last_par >> s) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        // One iteration = one stage (BK k) of one tile: 8 MMAs into the tile's
        // accumulator and one commit that frees the shared-memory stage (and,
        // A_SLOTS iterations later, the TMEM A slot: the unpack warps wait on the
        // same barrier). The tensor core queues only about one MMA ahead, so the
        // wait for the next iteration's operands is done before the last MMA
        // of this one is issued, while the queued MMAs still run. (Committing
        // behind the next iteration's first MMA instead was measured slower:
        // with two A slots it delays the unpack of the slot's next use.)
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_i8(BM, BT);
            constexpr int KSTEPS = BK / MMA_K;
            const int my_tiles = (num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
            const int total = my_tiles * num_kb;
            // ring positions of the current iteration (incremental: no divisions
            // on this thread, which paces the tensor core)
            int stage = 0, slot = 0, kb = 0, buf = 0;
            uint32_t sphase = 0, aphase = 0, bphase = 0;
            // The unpack warps arrive on aready only after their own wait on
            // full[] of the same iteration, so once aready has flipped the
            // TMA data of that iteration has landed as well: the MMA thread
            // waits on aready alone.
            bool ok = total > 0 ? ptx::mbar_wait(&sm.aready[0], 0, abort) : true;
            bool any = false;
            for (int it = 0; it < total && ok; ++it) {
                if (kb == 0) {
                    if (!ptx::mbar_wait(&sm.acc_empty[buf], bphase ^ 1u, abort)) break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)d_col<BT>(buf);
                const uint32_t a = tmem + (uint32_t)a_col<BT>(slot);
                const uint32_t b = ptx::smem_addr(sm.act[stage]);
                // k step kk reads the activation box kk / 4 at byte offset 32 (kk % 4)
                constexpr int KPB = XBOX / MMA_K;
#pragma unroll
                for (int kk = 0; kk < KSTEPS - 1; ++kk)
                    ptx::mma_i8_ts(d, a + kk * (MMA_K / 4),
                                   ptx::sdesc_k_sw128(b + (kk / KPB) * BT * XBOX + (kk % KPB) * MMA_K), idesc,
                                   (kb | kk) != 0);
                // next ring positions; wait for their operands while the MMAs
                // already queued keep the tensor core busy
                int nstage = stage + 1, nslot = slot + 1;
                uint32_t nsphase = sphase, naphase = aphase;
                if (nstage == STAGES) { nstage = 0; nsphase ^= 1u; }
                if (nslot == A_SLOTS) { nslot = 0; naphase ^= 1u; }
                const bool next_ok = it + 1 < total ? ptx::mbar_wait(&sm.aready[nslot], naphase, abort) : true;
                ptx::mma_i8_ts(d, a + (KSTEPS - 1) * (MMA_K / 4),
                               ptx::sdesc_k_sw128(b + ((KSTEPS - 1) / KPB) * BT * XBOX + ((KSTEPS - 1) % KPB) * MMA_K),
                               idesc, 1u);
                any = true;
                ptx::mma_commit(&sm.empty[stage]);
                if (++kb == num_kb) {
                    ptx::mma_commit(&sm.acc_full[buf]);
                    kb = 0;
                    if (++buf == 2) { buf = 0; bphase ^= 1u; }
                }
                stage = nstage; sphase = nsphase; slot = nslot; aphase = naphase;
                ok = next_ok;
            }
            if (any) {
                // All MMAs done before TMEM is released.
                ptx::mma_commit(&sm.mma_done);
                ptx::mbar_wait_drain(&sm.mma_done, 0);
            }
        }
    } else if (warp >= FIRST_UNPACK_WARP && warp < FIRST_EPI_WARP) {
        // ---------------------------------------------------- weight unpack
        // Thread r owns output-channel row r of the tile: 128 packed bytes per
        // stage, read from the 128B-swizzled tile (16-byte chunk c of row r
        // sits at chunk c ^ (r & 7)), expanded to 256 INT8 in k order and
        // stored to TMEM lane r, 64 columns (two stores of 32). Warpgroup wg
        // takes the pipeline iterations it with it % UNPACK_WG == wg.
        const int q = warp & 3;
        const int wg = (warp - FIRST_UNPACK_WARP) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        bool ok = true;
        int it = wg;  // this warpgroup's iterations: wg, wg + UNPACK_WG, ...
        const int total = ((num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * num_kb;
        for (; it < total && ok; it += UNPACK_WG) {
            {
                const int stage = it % STAGES;
                const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
                const int slot = it % A_SLOTS;
                const uint32_t aphase = (uint32_t)(it / A_SLOTS) & 1u;
                // every lane waits (each then sees the TMA data); the outcome is
                // made warp-uniform before the warp-collective tcgen05.st
                // the slot was last read by iteration it - A_SLOTS, whose MMAs
                // completed when that iteration's stage barrier flipped
                bool got = ptx::mbar_wait(&sm.full[stage], phase, abort);
                if (got && it >= A_SLOTS) {
                    const int j = it - A_SLOTS;
                    got = ptx::mbar_wait(&sm.empty[j % STAGES], (uint32_t)(j / STAGES) & 1u, abort);
                }
                (void)aphase;
                ok = __all_sync(0xffffffffu, got);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint8_t *row = sm.wpk[stage] + r * (BK / 2);
                const int sx_ = r & 7;
                if constexpr (UNPACK == UNPACK_NONE) {
                    // W8A8: row r of box `half` holds k in [128 half, +128)
                    // of the stage, 16-byte chunk c at chunk c ^ (r & 7)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint8_t *brow = sm.wpk[stage] + half * BM * XBOX + r * XBOX;
                        uint32_t out[32];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(brow + 16 * (c ^ sx_));
                            out[4 * c] = v.x;
                            out[4 * c + 1] = v.y;
                            out[4 * c + 2] = v.z;
                            out[4 * c + 3] = v.w;
                        }
                        ptx::tmem_st_32x32b_x32(tmem + lane_base + (uint32_t)(a_col<BT>(slot) + 32 * half), out);
                    }
                } else {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t out[32];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(row + 16 * ((4 * half + c) ^ sx_));
                            const uint32_t p[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                uint32_t lo, hi;  // lo = k0,k2,k4,k6; hi = k1,k3,k5,k7
                                if constexpr (UNPACK == UNPACK_SEXT) {
                                    unpack_s4x8(p[j], lo, hi);
                                } else {
                                    lo = (p[j] << 4) & 0xF0F0F0F0u;
                                    hi = p[j] & 0xF0F0F0F0u;
                                }
                                if constexpr (UNPACK == UNPACK_X16_PERM) {
                                    out[8 * c + 2 * j] = lo;
                                    out[8 * c + 2 * j + 1] = hi;
                                } else {
                                    out[8 * c + 2 * j] = __byte_perm(lo, hi, 0x5140);      // k0 k1 k2 k3
                                    out[8 * c + 2 * j + 1] = __byte_perm(lo, hi, 0x7362);  // k4 k5 k6 k7
                                }
                            }
                        }
                        ptx::tmem_st_32x32b_x32(tmem + lane_base + (uint32_t)(a_col<BT>(slot) + 32 * half), out);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sm.aready[slot]);
            }
        }
    } else if (warp >= FIRST_EPI_WARP) {
        // ---------------------------------------------------- epilogue
        // Thread owns output channel n (TMEM lane); per tile it first fills a
        // table of 1/sx for the tile's tokens (one entry per thread), then
        // dequantizes 32 tokens per tcgen05.ld.
        //
        // y = acc / (sx * sw) without a per-element division: with
        // r = (1/sx) * (1/sw), an approximation of 1/d for d = sx * sw, take
        // q0 = f * r and correct it once with the exact remainder,
        // q = q0 + (f - q0 * d) * r (two FMAs; Markstein's quotient
        // correction). The result is the correctly rounded quotient in
        // practice and always within a few ulp (<< 1e-6 relative).
        const int q = warp & 3;
        const int et = threadIdx.x - 32 * FIRST_EPI_WARP;  // 0..127
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int buf = 0;
        uint32_t acc_phase = 0;
        const unsigned fmt = flags & W4A8_OUT_MASK;
        const int epi_mode = fmt == W4A8_OUT_S32 ? 8
                             : (fmt == W4A8_OUT_BF16 ? 4 : 0) + (bias ? 2 : 0) + ((flags & W4A8_RELU) ? 1 : 0);
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int n_tile = tile / tiles_m, m_tile = tile % tiles_m;
            const int m_base = m_tile * BT;
            // reciprocal scales of this tile's tokens (the previous tile's
            // readers are past the named barrier at its end)
            for (int c = et; c < BT; c += 128) {
                const int m = m_base + c;
                const float v = m < M ? ld_dep(sx + m) : 1.0f;
                sm.tsx[c] = v;
                sm.rsx[c] = __frcp_rn(v);
                sm.trs[c] = (zpa.zp != nullptr && m < M) ? ld_dep_s32(zpa.rowsum + m) : 0;
            }
            // One decision for all four epilogue warps (this barrier also
            // publishes rsx): a warp that gave up must not leave the others
            // waiting at a named barrier.
            if (!ptx::bar_and(1, 128, ptx::mbar_wait(&sm.acc_full[buf], acc_phase, abort))) break;
            ptx::tc_fence_after();
            const int n = n_tile * BM + q * 32 + lane;
            const bool n_ok = n < N;
            const float swn = n_ok ? ld_dep(sw + n) : 1.0f;
            const float rswn = __frcp_rn(swn);
            const float bn = (bias && n_ok) ? ld_dep(bias + n) : 0.0f;
            const int32_t zpn = (zpa.zp != nullptr && n_ok) ? ld_dep_s32(zpa.zp + n) - 8 : 0;
#pragma unroll 1
            for (int c0 = 0; c0 < BT; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem + lane_base + (uint32_t)(d_col<BT>(buf) + c0), v);
                ptx::tmem_wait_ld();
                const int mrem = M - (m_base + c0);
                if (mrem <= 0) break;
                constexpr int SH = Cfg<BT, UNPACK>::SHIFT;
                const int m0 = m_base + c0;
                const float *tsx = sm.tsx + c0, *rsx = sm.rsx + c0;
                const int32_t *trs = sm.trs + c0;
#define W4A8_EPI(F, B, R) epi_chunk_any<F, B, R, SH>(v, Y, ldy, m0, mrem, n, n_ok, swn, rswn, bn, tsx, rsx, zpn, trs)
                switch (epi_mode) {
                    case 0: W4A8_EPI(EPI_F32, false, false); break;
                    case 1: W4A8_EPI(EPI_F32, false, true); break;
                    case 2: W4A8_EPI(EPI_F32, true, false); break;
                    case 3: W4A8_EPI(EPI_F32, true, true); break;
                    case 4: W4A8_EPI(EPI_BF16, false, false); break;
                    case 5: W4A8_EPI(EPI_BF16, false, true); break;
                    case 6: W4A8_EPI(EPI_BF16, true, false); break;
                    case 7: W4A8_EPI(EPI_BF16, true, true); break;
                    default: W4A8_EPI(EPI_S32, false, false); break;
                }
#undef W4A8_EPI
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.acc_empty[buf]);
            if (++buf == 2) { buf = 0; acc_phase ^= 1; }
            ptx::bar_sync(1, 128);  // rsx is rewritten next tile
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------- host side ---

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A 2-D byte tensor [rows][inner] with the given row stride; tiles of
// box_inner bytes x box_rows rows; out-of-range elements read as zero.
// 2-D tensor map: `inner` elements of `dtype` per row, `rows` rows `stride`
// bytes apart; boxes of box_inner x box_rows; reads outside are zero-filled.
inline bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner,
                        uint64_t rows, uint64_t stride, uint32_t box_inner, uint32_t box_rows,
                        CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {stride};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
inline bool make_map_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows, uint64_t stride,
                        uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
    return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, rows, stride, box_inner, box_rows, swz);
}

template <int BT, int UNPACK>
inline size_t smem_bytes() { return sizeof(Smem<BT, UNPACK>) + 1024; }

template <int BT, int UNPACK>
inline w4a8_status launch(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                          const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy, int sm_count,
                          cudaStream_t stream, ZpArgs zpa = ZpArgs{nullptr, nullptr}) {
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(k_gemm_tc<BT, UNPACK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem_bytes<BT, UNPACK>());
    });
    if (attr_err != cudaSuccess) return W4A8_ERR_CUDA;
    CUtensorMap tm_w, tm_x;
    // W8A8: Wp is the INT8 weight rows, ldp their stride in bytes
    const uint32_t w_box = Cfg<BT, UNPACK>::W8 ? XBOX : BK / 2;
    if (!make_map_u8(&tm_w, Wp, (uint64_t)ldp, (uint64_t)N, (uint64_t)ldp, w_box, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_u8(&tm_x, Xq, (uint64_t)ldq, (uint64_t)M, (uint64_t)ldq, XBOX, BT, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    const long long tiles = (long long)((M + BT - 1) / BT) * ((N + BM - 1) / BM);
    const int grid = (int)(tiles < sm_count ? tiles : sm_count);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem_bytes<BT, UNPACK>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_gemm_tc<BT, UNPACK>, tm_w, tm_x, M, N, K, sx, sw, bias, flags, Y, ldy,
                                       zpa);
    return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

}  // namespace tc

inline bool tc_supported(int M, int K, int N) {
    return M >= 1 && K >= 1 && N >= 1 && tc::encode_fn() != nullptr;
}

// act_perm: the INT8 activations use the k-permuted layout k_act_quant
// writes for this kernel (only inside w4a8_linear's workspace).
namespace tc {
// Token tile for a call: the one with the smallest estimated time, where a
// round of tiles over the SMs costs ceil(K / BK) iterations of about
// 8 x BT / 2 tensor cycles plus ~600 cycles of per-iteration overhead.
inline int pick_token_tile(int M, int N, int sm_count, bool w8 = false) {
    const int cand[4] = {192, 160, 128, 64};
    int best = w8 ? 160 : 192;
    long long best_cost = -1;
    for (int bt : cand) {
        if (bt == (w8 ? 192 : 160)) continue;  // INT4 forms: 192/128/64; W8A8: 160/128/64
        const long long tiles = (long long)((M + bt - 1) / bt) * ((N + BM - 1) / BM);
        const long long rounds = (tiles + sm_count - 1) / sm_count;
        const long long cost = rounds * (8LL * bt / 2 + 600);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bt;
        }
    }
    return best;
}

template <int UNPACK>
inline w4a8_status launch_bt(int bt, const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp,
                             int ldp, const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                             int sm_count, cudaStream_t stream, ZpArgs zpa) {
    if (bt == 64)
        return launch<64, UNPACK>(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, sm_count, stream, zpa);
    if (bt == 128)
        return launch<128, UNPACK>(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, sm_count, stream, zpa);
    return launch<192, UNPACK>(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, sm_count, stream, zpa);
}
}  // namespace tc

inline w4a8_status launch_gemm_tc(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp,
                                  int ldp, const float *sw, int N, const float *bias, unsigned flags, void *Y,
                                  int ldy, int sm_count, cudaStream_t stream, bool act_perm = false,
                                  ZpArgs zpa = ZpArgs{nullptr, nullptr}) {
    const int bt = tc::pick_token_tile(M, N, sm_count);
    if (K > tc::TC_X16_MAX_K) {
        if (act_perm) return W4A8_ERR_UNSUPPORTED;
        return tc::launch_bt<tc::UNPACK_SEXT>(bt, Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, sm_count,
                                              stream, zpa);
    }
    if (act_perm)
        return tc::launch_bt<tc::UNPACK_X16_PERM>(bt, Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy,
                                                  sm_count, stream, zpa);
    return tc::launch_bt<tc::UNPACK_X16>(bt, Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, sm_count,
                                         stream, zpa);
}

// W8A8 product on the tensor cores: Wq [N][ldw8] INT8 codes (ldw8 a multiple
// of 16, bytes k >= K zero), activations in natural k order.
inline w4a8_status launch_gemm_tc8(const int8_t *Xq, int M, int K, int ldq, const float *sx, const int8_t *Wq,
                                   int ldw8, const float *sw, int N, const float *bias, unsigned flags, void *Y,
                                   int ldy, int sm_count, cudaStream_t stream) {
    const int bt = tc::pick_token_tile(M, N, sm_count, true);
    const uint8_t *w = reinterpret_cast<const uint8_t *>(Wq);
    if (bt == 64)
        return tc::launch<64, tc::UNPACK_NONE>(Xq, M, K, ldq, sx, w, ldw8, sw, N, bias, flags, Y, ldy, sm_count, stream);
    if (bt == 128)
        return tc::launch<128, tc::UNPACK_NONE>(Xq, M, K, ldq, sx, w, ldw8, sw, N, bias, flags, Y, ldy, sm_count,
                                                stream);
    return tc::launch<160, tc::UNPACK_NONE>(Xq, M, K, ldq, sx, w, ldw8, sw, N, bias, flags, Y, ldy, sm_count, stream);
}

}  // namespace w4a8
