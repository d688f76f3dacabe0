// Tensor-core form of the group-wise INT4 product ("INT4" concept page,
// section 4.2, group quantization with group_size 128): per output channel n
// and group g of 128 consecutive k, a scale sa[n][g] and a zero point
// zp[n][g], and
//   y[m][n] = sum_g acc_g / (sx[m] * sa[n][g]),
//   acc_g   = sum_{k in g} xq[m][k] * (q[n][k] - zp[n][g])   (exact INT32),
// then bias and ReLU. The pipeline is the W4A8 tensor-core GEMM's (TMA
// stages of packed weights and INT8 activations, weights widened to INT8 in
// registers and written into TMEM as the MMA's A operand, tcgen05.mma
// kind::i8), with three changes:
//  * the weight warps widen each nibble to q - zp of its group (the stored
//    nibble is q - 8; sign-extend, then subtract zp - 8 byte-wise: values in
//    [-15, 15]), so a group's MMAs give acc_g itself, with no row sums;
//  * the MMA issuer starts a fresh INT32 accumulator for every group (a
//    group is one 128-k activation box: 4 MMAs) and alternates between two
//    accumulator buffers, committing each group to the epilogue;
//  * the epilogue drains every group: z += float(acc_g) * (1 / sa[n][g]) in
//    float32 registers, each warp on its own barrier wait (acc_g is at most 128 * 127 * 15 in size, exact in
//    float32), and at the end of the tile y = z * (1 / sx[m]), bias, ReLU.
// Factoring 1 / sx out of the group sum leaves one conversion and one FMA
// per output and group. The float32 result differs from a sequential sum of
// float(acc_g) / (sx * sa) by at most (ng + 3) * 2^-24 * sum_g |term_g|
// (rounded reciprocals, products, the sum and the final product), inside the
// (2 ng + 2) * 2^-24 * sum_g |term_g| bound of the group-wise layer.
//
// Warp roles (640 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs, warps 4-11 (two warpgroups taking pipeline iterations in
// turn) widen weights, warps 12-19 drain accumulators (warp 12 + e takes TMEM
// lanes 32 (e % 4).. and tokens 64 (e / 4)..). Every mbarrier wait is bounded.
#pragma once

#include "gemm_tc.cuh"

namespace w4a8 {
namespace tcg {

using tc::BK;
using tc::BM;
using tc::MMA_K;
using tc::XBOX;
constexpr int G = 128;                 // group size: one activation box of k
constexpr int BT = 128;                // tokens per tile (MMA N)
constexpr int STAGES = 4;              // 4 x 48 KB of shared memory
constexpr int A_SLOTS = 4;             // TMEM A slots of 64 columns
constexpr int A_COLS = BK / 4;
constexpr int UNPACK_WG = 2;
constexpr int FIRST_UNPACK_WARP = 4;
constexpr int FIRST_EPI_WARP = FIRST_UNPACK_WARP + 4 * UNPACK_WG;
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int NUM_THREADS = 32 * (FIRST_EPI_WARP + EPI_WARPS);
constexpr int TOK_PER_THREAD = BT / 2;
constexpr int TMEM_COLS = 512;
static_assert(BK == 2 * G && XBOX == G, "a pipeline iteration holds two groups, one activation box each");
static_assert(2 * BT + A_SLOTS * A_COLS <= TMEM_COLS, "TMEM budget");
static_assert(STAGES >= A_SLOTS && A_SLOTS % UNPACK_WG == 0, "A-slot reuse waits on a stage barrier");

__host__ __device__ constexpr int acc_col(int b) { return b * BT; }
__host__ __device__ constexpr int a_col(int slot) { return 2 * BT + slot * A_COLS; }

struct alignas(1024) Smem {
    uint8_t act[STAGES][BT * BK];      // two boxes of [BT][128 B], 128B-swizzled
    uint8_t wpk[STAGES][BM * BK / 2];  // [BM][128 B] packed, 128B-swizzled
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t aready[A_SLOTS];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    float rsx[BT];                     // 1 / sx of the tile's tokens
    uint32_t tmem_base;
    int abort;
};

// PERM: the INT8 activations are in the k-permuted layout of the activation
// pass (k0 k2 k4 k6 k1 k3 k5 k7 in every 8 k); otherwise natural order, and
// the widened weight bytes are permuted back to it.
template <bool PERM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_gemm_tc_grp(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, int M, int N,
              int K, int ng, const float *__restrict__ sx, const float *__restrict__ sa,
              const int32_t *__restrict__ zp, const float *__restrict__ bias, unsigned flags, void *__restrict__ Y,
              int ldy) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_kb = (K + BK - 1) / BK;
    const int tiles_m = (M + BT - 1) / BT;
    const int tiles_n = (N + BM - 1) / BM;
    const int num_tiles = tiles_m * tiles_n;
    const int my_tiles = (num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int total = my_tiles * num_kb;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < A_SLOTS; ++a) ptx::mbar_init(&sm.aready[a], 4);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&sm.acc_full[b], 1);
            ptx::mbar_init(&sm.acc_empty[b], EPI_WARPS);
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

    auto load_weights = [&](int stage, int n_tile, int kb) {
        ptx::mbar_arrive_expect_tx(&sm.full[stage], BT * BK + BM * BK / 2);
        ptx::tma_load_2d(sm.wpk[stage], &tm_w, kb * (BK / 2), n_tile * BM, &sm.full[stage]);
    };
    // static weights: the first stages' weight tiles before the dependency wait
    const int pre_w = (flags & W4A8_STATIC_WEIGHTS) ? min(STAGES, total) : 0;
    if (warp == 0 && lane == 0) {
        for (int it = 0; it < pre_w; ++it)
            load_weights(it, ((int)blockIdx.x + (it / num_kb) * (int)gridDim.x) / tiles_m, it % num_kb);
    }
    __syncwarp();
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0, it = 0;
            uint32_t phase = 0, issued = 0, last_par = 0;
            bool ok = true;
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
            if (!ok)
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s)) ptx::mbar_wait_drain(&sm.full[s], (last_par >> s) & 1u);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        // Per iteration (one stage, two groups): for each group that exists,
        // wait for a drained accumulator buffer, 4 MMAs starting from zero,
        // commit to the epilogue; then free the stage (and, A_SLOTS later, the
        // A slot).
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_i8(BM, BT);
            int stage = 0, slot = 0, kb = 0, gbuf = 0;
            uint32_t sphase = 0, aphase = 0, gphase = 0;
            bool ok = total > 0 ? ptx::mbar_wait(&sm.aready[0], 0, abort) : true;
            bool any = false;
            for (int it = 0; it < total && ok; ++it) {
                ptx::tc_fence_after();
                const uint32_t a = tmem + (uint32_t)a_col(slot);
                const uint32_t b = ptx::smem_addr(sm.act[stage]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (2 * kb + h >= ng) break;
                    if (!ptx::mbar_wait(&sm.acc_empty[gbuf], gphase ^ 1u, abort)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)acc_col(gbuf);
#pragma unroll
                    for (int kk = 0; kk < G / MMA_K; ++kk)
                        ptx::mma_i8_ts(d, a + (uint32_t)((G / MMA_K * h + kk) * (MMA_K / 4)),
                                       ptx::sdesc_k_sw128(b + h * BT * XBOX + kk * MMA_K), idesc, kk > 0 ? 1u : 0u);
                    ptx::mma_commit(&sm.acc_full[gbuf]);
                    any = true;
                    if (++gbuf == 2) { gbuf = 0; gphase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit(&sm.empty[stage]);
                if (++kb == num_kb) kb = 0;
                if (++stage == STAGES) { stage = 0; sphase ^= 1u; }
                if (++slot == A_SLOTS) { slot = 0; aphase ^= 1u; }
                if (it + 1 < total) ok = ptx::mbar_wait(&sm.aready[slot], aphase, abort);
            }
            (void)sphase;
            if (any) {
                ptx::mma_commit(&sm.mma_done);
                ptx::mbar_wait_drain(&sm.mma_done, 0);
            }
        }
    } else if (warp >= FIRST_UNPACK_WARP && warp < FIRST_EPI_WARP) {
        // ---------------------------------------------------- weight widening
        // Thread r owns channel row r of the tile: 128 packed bytes per stage
        // (chunk c of the swizzled row at chunk c ^ (r & 7)), two groups of
        // 128 k; each nibble becomes q - zp of its group as INT8, in the
        // k-permuted order of the activations (even k, then odd k, of every 8).
        const int q = warp & 3;
        const int wg = (warp - FIRST_UNPACK_WARP) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        bool ok = true;
        // the two groups' zero points of an iteration, fetched one iteration
        // of this warpgroup ahead so their latency hides behind the unpack
        auto zero_points = [&](int it, int32_t (&z)[2]) {
            const int kb = it % num_kb;
            const int tile = (int)blockIdx.x + (it / num_kb) * (int)gridDim.x;
            const int n = (tile / tiles_m) * BM + r;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int gi = 2 * kb + h;
                z[h] = (it < total && n < N && gi < ng) ? ld_dep_s32(zp + (size_t)n * ng + gi) - 8 : 0;
            }
        };
        int32_t z8_next[2];
        zero_points(wg, z8_next);
        for (int it = wg; it < total && ok; it += UNPACK_WG) {
            const int stage = it % STAGES;
            const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
            const int slot = it % A_SLOTS;
            const int kb = it % num_kb;
            const int32_t z8[2] = {z8_next[0], z8_next[1]};
            zero_points(it + UNPACK_WG, z8_next);
            bool got = ptx::mbar_wait(&sm.full[stage], phase, abort);
            if (got && it >= A_SLOTS) {
                const int j = it - A_SLOTS;
                got = ptx::mbar_wait(&sm.empty[j % STAGES], (uint32_t)(j / STAGES) & 1u, abort);
            }
            ok = __all_sync(0xffffffffu, got);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint8_t *row = sm.wpk[stage] + r * (BK / 2);
            const int sx_ = r & 7;
            // a pad nibble widens to 8 - zp, not 0: in the stage that holds
            // the end of K, bytes at k >= K are cleared, so whatever the INT8
            // rows hold there (w4g_linear_q allows anything) adds nothing
            const bool tail = (kb + 1) * BK > K;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t cc = ((uint32_t)z8[h] & 0xFFu) * 0x01010101u;
                uint32_t out[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + 16 * ((4 * h + c) ^ sx_));
                    const uint32_t p[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t lo, hi;  // lo = k0,k2,k4,k6; hi = k1,k3,k5,k7 (each q - 8)
                        unpack_s4x8(p[j], lo, hi);
                        lo = __vsub4(lo, cc);
                        hi = __vsub4(hi, cc);
                        if (tail) {
                            const int left = K - (kb * BK + G * h + 32 * c + 8 * j);  // k of this word still < K
                            uint32_t mlo = 0, mhi = 0;
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                mlo |= (2 * b < left ? 0xFFu : 0u) << (8 * b);
                                mhi |= (2 * b + 1 < left ? 0xFFu : 0u) << (8 * b);
                            }
                            lo &= mlo;
                            hi &= mhi;
                        }
                        if constexpr (PERM) {
                            out[8 * c + 2 * j] = lo;
                            out[8 * c + 2 * j + 1] = hi;
                        } else {
                            out[8 * c + 2 * j] = __byte_perm(lo, hi, 0x5140);      // k0 k1 k2 k3
                            out[8 * c + 2 * j + 1] = __byte_perm(lo, hi, 0x7362);  // k4 k5 k6 k7
                        }
                    }
                }
                ptx::tmem_st_32x32b_x32(tmem + lane_base + (uint32_t)(a_col(slot) + 32 * h), out);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.aready[slot]);
        }
    } else if (warp >= FIRST_EPI_WARP) {
        // ---------------------------------------------------- epilogue
        const int e = warp - FIRST_EPI_WARP;
        const int q = e & 3, half = e >> 2;
        const int et = e * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const unsigned fmt = flags & W4A8_OUT_MASK;
        const bool relu = (flags & W4A8_RELU) != 0;
        int gbuf = 0;
        uint32_t gphase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int n_tile = tile / tiles_m, m_tile = tile % tiles_m;
            const int m_base = m_tile * BT;
            for (int c = et; c < BT; c += EPI_THREADS) {
                const int m = m_base + c;
                sm.rsx[c] = __frcp_rn(m < M ? ld_dep(sx + m) : 1.0f);
            }
            // publishes rsx (the previous tile's readers are past the barrier
            // at its end)
            ptx::bar_sync(1, EPI_THREADS);
            const int n = n_tile * BM + q * 32 + lane;
            const bool n_ok = n < N;
            float z[TOK_PER_THREAD];
#pragma unroll
            for (int j = 0; j < TOK_PER_THREAD; ++j) z[j] = 0.0f;
            float rsa = n_ok ? __frcp_rn(ld_dep(sa + (size_t)n * ng)) : 0.0f;
            // Each warp drains its share of every group on its own (a
            // barrier of all eight warps per group cost more than the drain);
            // the warps agree on the outcome once per tile, below.
            for (int g = 0; g < ng; ++g) {
                const float rsa_next = (n_ok && g + 1 < ng) ? __frcp_rn(ld_dep(sa + (size_t)n * ng + g + 1)) : 0.0f;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&sm.acc_full[gbuf], gphase, abort))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                // 16 columns per TMEM load (z and one load fit the 96 registers
                // a thread of this 640-thread block gets)
#pragma unroll
                for (int c = 0; c < TOK_PER_THREAD / 16; ++c) {
                    uint32_t v[16];
                    ptx::tmem_ld_32x32b_x16(
                        tmem + lane_base + (uint32_t)(acc_col(gbuf) + TOK_PER_THREAD * half + 16 * c), v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        z[16 * c + j] = __fmaf_rn(__int2float_rn((int32_t)v[j]), rsa, z[16 * c + j]);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sm.acc_empty[gbuf]);
                if (++gbuf == 2) { gbuf = 0; gphase ^= 1u; }
                rsa = rsa_next;
            }
            // one decision for all epilogue warps: a warp that gave up must not
            // leave the others waiting at the named barriers
            if (!ptx::bar_and(1, EPI_THREADS, ok)) break;
            const float bn = (bias != nullptr && n_ok) ? ld_dep(bias + n) : 0.0f;
#pragma unroll
            for (int j = 0; j < TOK_PER_THREAD; ++j) {
                const int c = TOK_PER_THREAD * half + j;
                const int m = m_base + c;
                if (m >= M || !n_ok) continue;
                float y = __fmul_rn(z[j], sm.rsx[c]);
                if (bias != nullptr) y = __fadd_rn(y, bn);
                if (relu) y = y > 0.0f ? y : 0.0f;
                const size_t off = (size_t)m * (size_t)ldy + (size_t)n;
                if (fmt == W4A8_OUT_BF16)
                    static_cast<__nv_bfloat16 *>(Y)[off] = __float2bfloat16_rn(y);
                else
                    static_cast<float *>(Y)[off] = y;
            }
            ptx::bar_sync(1, EPI_THREADS);  // rsx is rewritten next tile
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

inline size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Xq: INT8 rows (k-permuted layout of k_act_quant with PERM, or natural
// order), ldq a multiple of 16. Wp: the zero-point storage (nibbles q - 8), ldp a multiple
// of 16. sa, zp: [N][ng]. Output f32 or bf16.
template <bool PERM>
inline w4a8_status launch(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                          const float *sa, const int32_t *zp, int ng, int N, const float *bias, unsigned flags,
                          void *Y, int ldy, int sm_count, cudaStream_t stream) {
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(k_gemm_tc_grp<PERM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem_bytes());
    });
    if (attr_err != cudaSuccess) return W4A8_ERR_CUDA;
    CUtensorMap tm_w, tm_x;
    if (!tc::make_map_u8(&tm_w, Wp, (uint64_t)ldp, (uint64_t)N, (uint64_t)ldp, BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tc::make_map_u8(&tm_x, Xq, (uint64_t)ldq, (uint64_t)M, (uint64_t)ldq, XBOX, BT, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    const long long tiles = (long long)((M + BT - 1) / BT) * ((N + BM - 1) / BM);
    const int grid = (int)(tiles < sm_count ? tiles : sm_count);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e =
        cudaLaunchKernelEx(&cfg, k_gemm_tc_grp<PERM>, tm_w, tm_x, M, N, K, ng, sx, sa, zp, bias, flags, Y, ldy);
    return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

}  // namespace tcg
}  // namespace w4a8
