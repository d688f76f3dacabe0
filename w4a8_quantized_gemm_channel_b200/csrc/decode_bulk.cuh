// Persistent decode kernel: the weight stream staged through shared memory by
// the tensor-memory-access (TMA) engine (steps 4-6 of "How it works" in the
// Keras guide "INT4 quantization in Keras", for at most 8 activation rows).
//
// With few activation rows the layer is a stream of the packed weights, and
// on B200 an SM needs well over 100 KB of loads in flight to draw its share
// of HBM bandwidth (the loaded latency is several microseconds). A block is
// persistent: a producer thread keeps a ring of up to 8 stages full - a stage
// is one 2-D TMA copy of 16 packed rows x up to 2048 bytes (4096 k),
// zero-filled past the row's packed bytes and past N - sized to the shared
// memory left next to the activation rows, and the block walks its 16-channel
// groups g = blockIdx.x, + gridDim.x, ... through that one ring. Long layers
// run two such blocks per SM (two independent streams per SM measured
// faster than one with twice the ring). A short layer holds its whole share
// of the weights in the ring and leaves room on every SM for the blocks of
// the next launch, whose copies are then on the way before this one finishes
// (programmatic dependent launch).
//
// The 8 consumer warps first bring the INT8 activation rows into shared
// memory - copied from Xq, or quantized from X in the block (FUSED) - in a
// k-permuted order: inside every 8 consecutive k the bytes sit as
// k0 k2 k4 k6 k1 k3 k5 k7, which is the order in which the nibble unpack
// yields weight codes, so no byte shuffles remain in the inner loop. Consumer
// warp w takes the 64-byte chunks c = w, w + 8, ... of every stage (k in
// [2 sb s + 128 c, +128) for stage s of sb bytes per row); thread (g, t)
// multiplies bytes 16t..16t+15 of rows g and g + 8 with the activation bytes
// of the same k on the legacy integer tensor-core path (mma.sync m16n8k32).
// Nibbles are kept in the high half of their byte (16 q, two logic ops per
// word): the sum is 16 x the product and is shifted back exactly. That needs
// 128 * 127 * K < 2^31, so the kernel serves K <= X16_MAX_K.
//
// Every mbarrier wait is bounded; a wait that runs out sets the block's abort
// flag and the device status word, the other waits then give up, the block
// writes no further output, and the producer waits for its copies in flight
// before the block exits.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "linear_simt.cuh"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace dbulk {

constexpr int CONSUMER_WARPS = 8;
constexpr int THREADS = (CONSUMER_WARPS + 1) * 32;
constexpr int CONSUMERS = CONSUMER_WARPS * 32;
constexpr int ROWS = 16;               // output channels per group
constexpr int TOK = 8;                 // activation rows (one tile: M <= 8)
constexpr int MAX_STAGE_BYTES = 2048;  // packed bytes of a row per stage: a box of 256 x 8 bytes
constexpr int MAX_RING = 8;            // ring slots (mbarrier pairs)
constexpr int SMEM_BUDGET = 100 * 1024;  // ring + activation rows of one block: two blocks per SM
constexpr int SM_SMEM = 220 * 1024;      // what blocks may take of an SM's shared memory
constexpr int X16_MAX_K = 131072;

// Stage geometry of a K (host and device agree on it).
struct Geometry {
    int kp;     // packed bytes of a row that hold codes (16-aligned)
    int sb;     // packed bytes of a row per stage (multiple of 64)
    int nst;    // stages per group
    int pitch;  // activation row pitch in shared memory: all k of the stages + 16
    __host__ __device__ explicit Geometry(int K) {
        kp = packed_row_bytes(K);
        const int kp64 = (kp + 63) / 64 * 64;
        sb = kp64 < MAX_STAGE_BYTES ? kp64 : MAX_STAGE_BYTES;
        nst = (kp + sb - 1) / sb;
        pitch = 2 * sb * nst + 16;
    }
    __host__ __device__ int stage_bytes() const { return ROWS * sb; }
    __host__ __device__ size_t xs_bytes(int rows) const { return (size_t)rows * pitch; }
};

struct Smem {
    uint64_t full[MAX_RING];
    uint64_t empty[MAX_RING];
    int32_t red[CONSUMER_WARPS][ROWS][TOK + 1];
    float part[TOK][CONSUMER_WARPS];
    float sxs[TOK];
    int abort;
};

// Codes of 8 consecutive k (v[0..7] at k0..k0+7, scale s) in the permuted
// order: word 0 = k0 k2 k4 k6, word 1 = k1 k3 k5 k7 (codes past K are 0).
__device__ __forceinline__ uint2 act_codes8_perm(const float (&v)[8], float s, int k0, int K) {
    uint32_t even = 0, odd = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        even |= act_code8(v[2 * b], s, k0 + 2 * b < K) << (8 * b);
        odd |= act_code8(v[2 * b + 1], s, k0 + 2 * b + 1 < K) << (8 * b);
    }
    return make_uint2(even, odd);
}

// Quantize activation rows 0..rows-1 of X (step 3, the arithmetic of
// k_act_quant, so the same codes and scales) into xs [rows][pitch] (permuted
// order) and sm.sxs, by the CONSUMERS threads. Each thread keeps J8 units of
// 8 floats of every row in registers between the abs-max and the code pass
// (ks <= 8 * CONSUMERS * J8).
template <int R, int J8>
__device__ __forceinline__ void quantize_rows(const float *X, int ldx, int vec4, int rows, int K, int ks,
                                              int pitch, int8_t *xs, Smem &sm, int tid, int lane, int warp) {
    float v[R][J8][8];
    float am[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        am[r] = 0.0f;
#pragma unroll
        for (int j = 0; j < J8; ++j) {
            const int k = 8 * (tid + CONSUMERS * j);
#pragma unroll
            for (int b = 0; b < 8; ++b) v[r][j][b] = 0.0f;
            if (r < rows && k < K) {
                const float *x = X + (size_t)r * ldx + k;
                if (vec4 && k + 7 < K) {
                    const float4 f0 = ld_dep_f4(x), f1 = ld_dep_f4(x + 4);
                    v[r][j][0] = f0.x; v[r][j][1] = f0.y; v[r][j][2] = f0.z; v[r][j][3] = f0.w;
                    v[r][j][4] = f1.x; v[r][j][5] = f1.y; v[r][j][6] = f1.z; v[r][j][7] = f1.w;
                } else {
#pragma unroll
                    for (int b = 0; b < 8; ++b)
                        if (k + b < K) v[r][j][b] = ld_dep(x + b);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int j = 0; j < J8; ++j)
#pragma unroll
            for (int b = 0; b < 8; ++b) am[r] = fmaxf(am[r], fabsf(v[r][j][b]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am[r] = fmaxf(am[r], __shfl_xor_sync(0xffffffffu, am[r], o));
        if (lane == 0) sm.part[r][warp] = am[r];
    }
    ptx::bar_sync(1, CONSUMERS);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (r >= rows) continue;
        float a = sm.part[r][0];
#pragma unroll
        for (int w = 1; w < CONSUMER_WARPS; ++w) a = fmaxf(a, sm.part[r][w]);
        const float s = act_scale_from_amax(a);
        if (tid == 0) sm.sxs[r] = s;
#pragma unroll
        for (int j = 0; j < J8; ++j) {
            const int k = 8 * (tid + CONSUMERS * j);
            if (k < ks) *reinterpret_cast<uint2 *>(xs + r * pitch + k) = act_codes8_perm(v[r][j], s, k, K);
        }
    }
    ptx::bar_sync(1, CONSUMERS);
}

// The same quantization for rows whose values do not fit the registers (any
// K the stages cover): pass 1 reduces each row's abs-max while streaming X
// (up to 4 units of 8 floats per row in flight per thread), pass 2 reads X
// again - L1/L2-resident by then - and writes the codes.
template <int R>
__device__ __forceinline__ void quantize_rows_2pass(const float *X, int ldx, int vec4, int rows, int K, int ks,
                                                    int pitch, int8_t *xs, Smem &sm, int tid, int lane, int warp) {
    float am[R];
#pragma unroll
    for (int r = 0; r < R; ++r) am[r] = 0.0f;
    auto load8 = [&](int r, int k, float (&v)[8]) {
#pragma unroll
        for (int b = 0; b < 8; ++b) v[b] = 0.0f;
        if (r >= rows || k >= K) return;
        const float *x = X + (size_t)r * ldx + k;
        if (vec4 && k + 7 < K) {
            const float4 f0 = ld_dep_f4(x), f1 = ld_dep_f4(x + 4);
            v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
            v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
        } else {
#pragma unroll
            for (int b = 0; b < 8; ++b)
                if (k + b < K) v[b] = ld_dep(x + b);
        }
    };
    constexpr int UNR = R >= 4 ? 1 : 4 / R;  // units per row in flight
    for (int k0 = 8 * tid; k0 < K; k0 += 8 * CONSUMERS * UNR) {
        float v[UNR][R][8];
#pragma unroll
        for (int u = 0; u < UNR; ++u)
#pragma unroll
            for (int r = 0; r < R; ++r) load8(r, k0 + 8 * CONSUMERS * u, v[u][r]);
#pragma unroll
        for (int u = 0; u < UNR; ++u)
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int b = 0; b < 8; ++b) am[r] = fmaxf(am[r], fabsf(v[u][r][b]));
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am[r] = fmaxf(am[r], __shfl_xor_sync(0xffffffffu, am[r], o));
        if (lane == 0) sm.part[r][warp] = am[r];
    }
    ptx::bar_sync(1, CONSUMERS);
    float sc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float a = sm.part[r][0];
#pragma unroll
        for (int w = 1; w < CONSUMER_WARPS; ++w) a = fmaxf(a, sm.part[r][w]);
        sc[r] = act_scale_from_amax(a);
        if (tid == 0 && r < rows) sm.sxs[r] = sc[r];
    }
    for (int k0 = 8 * tid; k0 < ks; k0 += 8 * CONSUMERS * UNR) {
        float v[UNR][R][8];
#pragma unroll
        for (int u = 0; u < UNR; ++u)
#pragma unroll
            for (int r = 0; r < R; ++r) load8(r, k0 + 8 * CONSUMERS * u, v[u][r]);
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int k = k0 + 8 * CONSUMERS * u;
            if (k >= ks) continue;
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (r < rows) *reinterpret_cast<uint2 *>(xs + r * pitch + k) = act_codes8_perm(v[u][r], sc[r], k, K);
        }
    }
    ptx::bar_sync(1, CONSUMERS);
}

// Copy INT8 activation rows (natural order, row stride ldq) into xs in the
// permuted order, 16 bytes per load; k from min(ldq, ks) on reads as 0.
__device__ __forceinline__ void stage_rows(const int8_t *Xq, int ldq, int rows, int ks, int pitch, int8_t *xs,
                                           int tid) {
    const int per = ks / 16, have = min(ldq, ks) / 16;
#pragma unroll 4
    for (int i = tid; i < rows * per; i += CONSUMERS) {
        const int r = i / per, c = i - r * per;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (c < have) {
            const uint4 x = ld_dep_v4(Xq + (size_t)r * ldq + 16 * c);
            v = make_uint4(__byte_perm(x.x, x.y, 0x6420), __byte_perm(x.x, x.y, 0x7531),
                           __byte_perm(x.z, x.w, 0x6420), __byte_perm(x.z, x.w, 0x7531));
        }
        *reinterpret_cast<uint4 *>(xs + r * pitch + 16 * c) = v;
    }
    ptx::bar_sync(1, CONSUMERS);
}

// MMAs of one stage: this warp's 64-byte chunks c = warp, warp + 8, ... of
// the 16 rows x sb bytes at `st` (already offset by 16 t) against the INT8
// rows (xrow = this thread's row g at byte 32 t; stage s covers
// k in [2 sb s, 2 sb (s + 1))). Four accumulators (one per word of a piece)
// keep the MMAs in four short dependency chains.
__device__ __forceinline__ void stage_mma(int32_t (&acc)[4][4], const uint8_t *st, int sb, int s,
                                          const int8_t *xrow, bool x_ok, int g, int warp) {
    const int cps = sb / 64;
#pragma unroll 2
    for (int c = warp; c < cps; c += CONSUMER_WARPS) {
        const uint4 wa = ptx::lds128(st + g * sb + 64 * c);
        const uint4 wb = ptx::lds128(st + (g + 8) * sb + 64 * c);
        const int8_t *xp = xrow + 2 * sb * s + 128 * c;
        const uint4 x0 = x_ok ? ptx::lds128(xp) : make_uint4(0, 0, 0, 0);
        const uint4 x1 = x_ok ? ptx::lds128(xp + 16) : make_uint4(0, 0, 0, 0);
        const uint32_t pa[4] = {wa.x, wa.y, wa.z, wa.w}, pb[4] = {wb.x, wb.y, wb.z, wb.w};
        const uint32_t xe[4] = {x0.x, x0.z, x1.x, x1.z}, xo[4] = {x0.y, x0.w, x1.y, x1.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t alo = (pa[q] << 4) & 0xF0F0F0F0u;  // 16 q of even k
            const uint32_t ahi = pa[q] & 0xF0F0F0F0u;         // 16 q of odd k
            const uint32_t blo = (pb[q] << 4) & 0xF0F0F0F0u;
            const uint32_t bhi = pb[q] & 0xF0F0F0F0u;
            mma_s8_16832(acc[q], alo, blo, ahi, bhi, xe[q], xo[q]);
        }
    }
}

// End of a 16-channel group: the warps' C fragments (rows g, g+8 = channels,
// columns 2t, 2t+1 = tokens) meet in shared memory; thread e (< 16 x TOK)
// gets the block total of output (channel e % 16, token e / 16), as 16 x the
// product (returned shifted back). Returns false, after raising the abort
// flag, if any consumer warp gave up; every consumer thread then agrees.
__device__ __forceinline__ bool group_reduce(Smem &sm, int32_t (&acc)[4][4], bool ok, int warp, int g, int t,
                                             volatile int *abort, int32_t &sum) {
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[0][q] += acc[1][q] + acc[2][q] + acc[3][q];
    sm.red[warp][g][2 * t] = acc[0][0];
    sm.red[warp][g][2 * t + 1] = acc[0][1];
    sm.red[warp][g + 8][2 * t] = acc[0][2];
    sm.red[warp][g + 8][2 * t + 1] = acc[0][3];
    if (!ptx::bar_and(1, CONSUMERS, ok)) {
        if (threadIdx.x == 0) *abort = 1;  // lets the producer stop refilling
        return false;
    }
    sum = 0;
    if (threadIdx.x < 16 * TOK) {
#pragma unroll
        for (int w = 0; w < CONSUMER_WARPS; ++w) sum += sm.red[w][threadIdx.x % 16][threadIdx.x / 16];
        sum >>= 4;  // exact: every term is a multiple of 16
    }
    return true;
}

// tm_w: the packed weights as a [N][kp / 8] tensor of 8-byte elements with
// row stride ldp, boxes of sb / 8 x 16. ring_n: ring slots (the host sizes
// the dynamic shared memory as ring_n stages + the activation rows).
// EARLY: the weights are final at launch (behind the activation pass, or
// W4A8_STATIC_WEIGHTS), so the ring is filled before the dependency wait;
// otherwise the first stages are only prefetched into L2 before it.
// FUSED: the block quantizes X itself (M <= R): with the values held in
// registers when ks <= 2048 J8, in two passes over X when J8 = 0; otherwise
// Xq / sx come from the activation pass or the caller.
template <bool EARLY, bool FUSED, int R, int J8>
__global__ void __launch_bounds__(THREADS, 3)
k_decode_ring(const __grid_constant__ CUtensorMap tm_w, const int8_t *Xq, int ldq, const float *sx,
              const float *X, int ldx, int vec4, int M, int K, const float *sw, int N,
              const float *bias, unsigned flags, void *Y, int ldy, int ring_n, ZpArgs zpa) {
    __shared__ Smem sm;
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    const Geometry geo(K);
    const int sb = geo.sb, nst = geo.nst, pitch = geo.pitch, stage_bytes = geo.stage_bytes();
    const int ks = pitch - 16;  // k covered by the stages
    uint8_t *ring = dyn_smem;   // [ring_n][16][sb]
    int8_t *xs = reinterpret_cast<int8_t *>(dyn_smem + (size_t)ring_n * stage_bytes);  // [rows][pitch]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int groups = (N + ROWS - 1) / ROWS;
    const int my_groups = (groups - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int items = my_groups * nst;  // (group, stage) pairs of this block
    const int rows = min(TOK, M);
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ring_n; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], CONSUMER_WARPS);
        }
        sm.abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    griddep_launch_dependents();

    if (warp == CONSUMER_WARPS) {
        // ------------------------------------------------- producer (lane 0)
        int issued = 0;
        auto issue = [&](int it) {
            const int j = it / nst, s = it - j * nst;
            const int slot = it % ring_n;
            ptx::mbar_arrive_expect_tx(&sm.full[slot], (uint32_t)stage_bytes);
            ptx::tma_load_2d(ring + (size_t)slot * stage_bytes, &tm_w, s * (sb / 8),
                             ((int)blockIdx.x + j * (int)gridDim.x) * ROWS, &sm.full[slot]);
            ++issued;
        };
        const int pre = min(ring_n, items);
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_w);
            if constexpr (EARLY) {
                for (int it = 0; it < pre; ++it) issue(it);
            } else {
                for (int it = 0; it < pre; ++it) {
                    const int j = it / nst, s = it - j * nst;
                    ptx::tma_prefetch_2d(&tm_w, s * (sb / 8), ((int)blockIdx.x + j * (int)gridDim.x) * ROWS);
                }
            }
        }
        // The whole warp waits together: a lane blocked in griddepcontrol.wait
        // holds its warp, so lane 0 must have issued the copies above first.
        __syncwarp();
        griddep_wait();
        if (lane != 0) return;
        if constexpr (!EARLY) {
            for (int it = 0; it < pre; ++it) issue(it);
        }
        for (int it = ring_n; it < items; ++it) {
            // the slot is free once every consumer warp arrived on its last use
            if (!ptx::mbar_wait(&sm.empty[it % ring_n], (uint32_t)(it / ring_n - 1) & 1u, abort)) break;
            issue(it);
        }
        // the block may exit only when every copy it issued has landed
        for (int it = max(0, issued - ring_n); it < issued; ++it)
            ptx::mbar_wait_drain(&sm.full[it % ring_n], (uint32_t)(it / ring_n) & 1u);
        return;
    }

    // -------------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    const int e_ch = threadIdx.x % 16, e_tk = threadIdx.x / 16;
    const bool e_row = threadIdx.x < 16 * TOK && e_tk < rows;
    const bool has_bias = bias != nullptr && (flags & W4A8_OUT_MASK) != W4A8_OUT_S32;
    griddep_wait();
    float e_sx = 1.0f;
    if constexpr (FUSED) {
        if constexpr (J8 > 0)
            quantize_rows<R, J8>(X, ldx, vec4, rows, K, ks, pitch, xs, sm, threadIdx.x, lane, warp);
        else
            quantize_rows_2pass<R>(X, ldx, vec4, rows, K, ks, pitch, xs, sm, threadIdx.x, lane, warp);
        if (e_row) e_sx = sm.sxs[e_tk];
    } else {
        if (e_row) e_sx = ld_dep(sx + e_tk);
        stage_rows(Xq, ldq, rows, ks, pitch, xs, threadIdx.x);
    }

    const bool x_ok = g < rows;
    const int8_t *xrow = xs + g * pitch + 32 * t;
    bool ok = true;
    for (int j = 0; j < my_groups; ++j) {
        const int n0 = ((int)blockIdx.x + j * (int)gridDim.x) * ROWS;
        const bool e_ok = e_row && n0 + e_ch < N;
        float e_sw = 1.0f, e_b = 0.0f;
        if (e_ok) {  // needed after the group's MMAs: the loads overlap them
            e_sw = ld_dep(sw + n0 + e_ch);
            if (has_bias) e_b = ld_dep(bias + n0 + e_ch);
        }
        int32_t acc[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
        for (int s = 0; s < nst && ok; ++s) {
            const int it = j * nst + s, slot = it % ring_n;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&sm.full[slot], (uint32_t)(it / ring_n) & 1u, abort))) {
                ok = false;  // warp-uniform, so the warp leaves the loop together
                break;
            }
            stage_mma(acc, ring + (size_t)slot * stage_bytes + 16 * t, sb, s, xrow, x_ok, g, warp);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.empty[slot]);
        }
        int32_t sum;
        if (!group_reduce(sm, acc, ok, warp, g, t, abort, sum)) return;
        if (e_ok)
            store_value(Y, ldy, e_tk, n0 + e_ch, zp_fix(sum, zpa, e_tk, n0 + e_ch), e_sx, e_sw, has_bias, e_b, flags);
        ptx::bar_sync(1, CONSUMERS);  // red is rewritten by the next group
    }
}

// ---------------------------------------------------------------------------
// Grouped decode: many independent few-row linears in one persistent launch.
// The problems' 16-channel groups are numbered one after another; block b
// takes a contiguous run of them holding 1 / grid of all weight bytes, so it
// switches problems rarely and the blocks finish together. Its producer streams every (group, stage) of
// that run through one ring (slots of the largest stage, 16 x 2048 bytes)
// with each problem's own tensor map; its consumers quantize a problem's
// activation rows into shared memory (two passes over X, the arithmetic of
// k_act_quant) whenever the run enters that problem, then multiply as in
// k_decode_ring. Each problem's result is the same bits a single call gives.
// The table travels by value in the launch parameters (tensor maps
// included), so a captured graph holds everything it needs.
// ---------------------------------------------------------------------------
constexpr int MAX_GROUPED = 64;
constexpr int GROUPED_SLOT = ROWS * MAX_STAGE_BYTES;

struct GroupedProblem {
    CUtensorMap tm;  // packed weights as [N][kp / 8] elements of 8 bytes (boxes of sb / 8 x 16)
    const float *X;
    const float *sw;
    const float *bias;
    void *Y;
    int M, K, ldx, ldy, N, vec4, group0, pad;
    long long bytes0;     // packed weight bytes of all earlier problems' groups
    long long group_bytes;  // packed weight bytes of one of this problem's groups
};
struct GroupedTable {
    GroupedProblem p[MAX_GROUPED];
    int count;
    int total_groups;
    long long total_bytes;
};

// The first group whose weights start at or after byte `b` of the run of all
// groups (blocks split the work by weight bytes, not by group count: a group
// of a long-K layer carries several times the bytes of a short one).
__device__ __forceinline__ int grouped_first_group(const GroupedTable &tab, long long b) {
    int p = 0;
    while (p + 1 < tab.count && tab.p[p + 1].bytes0 <= b) ++p;
    const GroupedProblem &q = tab.p[p];
    const long long off = b - q.bytes0;
    const int ng = (q.N + ROWS - 1) / ROWS;
    int j = (int)((off + q.group_bytes - 1) / q.group_bytes);
    if (j > ng) j = ng;
    return q.group0 + j;
}
static_assert(sizeof(GroupedTable) <= 30 * 1024, "kernel parameter space");

// Position in a block's run of (group, stage) items.
struct GroupedCursor {
    int gi, p, s, nst, sb;
    __device__ __forceinline__ void enter(const GroupedTable &tab) {
        while (p + 1 < tab.count && gi >= tab.p[p + 1].group0) ++p;
        const Geometry geo(tab.p[p].K);
        nst = geo.nst;
        sb = geo.sb;
    }
    __device__ __forceinline__ void next(const GroupedTable &tab) {
        if (++s == nst) {
            s = 0;
            ++gi;
            enter(tab);
        }
    }
};

template <bool EARLY, int R>
__global__ void __launch_bounds__(THREADS, 2)
k_decode_grouped(const __grid_constant__ GroupedTable tab, unsigned flags, int ring_n) {
    __shared__ Smem sm;
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t *ring = dyn_smem;  // [ring_n][GROUPED_SLOT]
    int8_t *xs = reinterpret_cast<int8_t *>(dyn_smem + (size_t)ring_n * GROUPED_SLOT);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long B = tab.total_bytes;
    const int g_begin = grouped_first_group(tab, B * blockIdx.x / gridDim.x);
    const int g_end = blockIdx.x + 1 == gridDim.x ? tab.total_groups
                                                    : grouped_first_group(tab, B * (blockIdx.x + 1) / gridDim.x);
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ring_n; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], CONSUMER_WARPS);
        }
        sm.abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    griddep_launch_dependents();
    if (g_begin >= g_end) {
        griddep_wait();
        return;
    }

    if (warp == CONSUMER_WARPS) {
        // ------------------------------------------------- producer (lane 0)
        GroupedCursor cur{g_begin, 0, 0, 0, 0};
        if (lane == 0) cur.enter(tab);
        int issued = 0;
        auto issue = [&]() {
            const GroupedProblem &pr = tab.p[cur.p];
            const int slot = issued % ring_n;
            ptx::mbar_arrive_expect_tx(&sm.full[slot], (uint32_t)(ROWS * cur.sb));
            ptx::tma_load_2d(ring + (size_t)slot * GROUPED_SLOT, &pr.tm, cur.s * (cur.sb / 8),
                             (cur.gi - pr.group0) * ROWS, &sm.full[slot]);
            ++issued;
            cur.next(tab);
        };
        if constexpr (EARLY) {
            if (lane == 0)
                while (issued < ring_n && cur.gi < g_end) issue();
        }
        // the whole warp waits together (a lane in griddepcontrol.wait holds it)
        __syncwarp();
        griddep_wait();
        if (lane != 0) return;
        bool ok = true;
        while (ok && cur.gi < g_end) {
            if (issued >= ring_n) {
                const int j = issued - ring_n;  // last use of this slot
                ok = ptx::mbar_wait(&sm.empty[j % ring_n], (uint32_t)(j / ring_n) & 1u, abort);
                if (!ok) break;
            }
            issue();
        }
        // the block may exit only when every copy it issued has landed
        for (int it = max(0, issued - ring_n); it < issued; ++it)
            ptx::mbar_wait_drain(&sm.full[it % ring_n], (uint32_t)(it / ring_n) & 1u);
        return;
    }

    // -------------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    const int e_ch = threadIdx.x % 16, e_tk = threadIdx.x / 16;
    const bool out_s32 = (flags & W4A8_OUT_MASK) == W4A8_OUT_S32;
    griddep_wait();
    GroupedCursor cur{g_begin, 0, 0, 0, 0};
    cur.enter(tab);
    int staged = -1, item = 0;
    bool ok = true;
    float e_sx = 1.0f;
    while (cur.gi < g_end) {
        const GroupedProblem &pr = tab.p[cur.p];
        const Geometry geo(pr.K);
        const int rows = pr.M;
        if (cur.p != staged) {  // the run enters a new problem: its INT8 rows
            quantize_rows_2pass<R>(pr.X, pr.ldx, pr.vec4, rows, pr.K, geo.pitch - 16, geo.pitch, xs, sm,
                                   threadIdx.x, lane, warp);
            staged = cur.p;
            e_sx = (threadIdx.x < 16 * TOK && e_tk < rows) ? sm.sxs[e_tk] : 1.0f;
        }
        const int n0 = (cur.gi - pr.group0) * ROWS;
        const bool e_ok = threadIdx.x < 16 * TOK && e_tk < rows && n0 + e_ch < pr.N;
        const bool has_bias = pr.bias != nullptr && !out_s32;
        float e_sw = 1.0f, e_b = 0.0f;
        if (e_ok) {
            e_sw = ld_dep(pr.sw + n0 + e_ch);
            if (has_bias) e_b = ld_dep(pr.bias + n0 + e_ch);
        }
        int32_t acc[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
        const int8_t *xrow = xs + g * geo.pitch + 32 * t;
        const int gi = cur.gi;
        while (ok && cur.gi == gi) {
            const int slot = item % ring_n;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&sm.full[slot], (uint32_t)(item / ring_n) & 1u, abort))) {
                ok = false;  // warp-uniform, so the warp leaves the loop together
                break;
            }
            stage_mma(acc, ring + (size_t)slot * GROUPED_SLOT + 16 * t, cur.sb, cur.s, xrow, g < rows, g, warp);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.empty[slot]);
            ++item;
            cur.next(tab);
        }
        int32_t sum;
        if (!group_reduce(sm, acc, ok, warp, g, t, abort, sum)) return;
        if (e_ok) store_value(pr.Y, pr.ldy, e_tk, n0 + e_ch, sum, e_sx, e_sw, has_bias, e_b, flags);
        ptx::bar_sync(1, CONSUMERS);  // red (and xs, on a problem change) are rewritten next
    }
}

}  // namespace dbulk
}  // namespace w4a8
