// CUDA-core paths of the quantized product (steps 4-6 of "How it works" in the
// Keras guide "INT4 quantization in Keras"): unpack INT4 -> INT8, INT8 x INT8
// accumulated in INT32, dequantize acc / (sx * sw), bias, ReLU.
//
//  * k_linear_generic: one thread per output, any shape; used for tiny layers.
//  * k_linear_decode : few activation rows (<= 16 per tile). The layer is then
//    bound by streaming the packed weights from HBM, so each warp issues its
//    16-byte weight loads up front and reduces them on the legacy integer
//    tensor-core path (mma.sync m16n8k32 s8): the FLOPs are tiny, what matters
//    is bytes in flight and few instructions per weight byte.
#pragma once

#include "common.cuh"

namespace w4a8 {

// ---------------------------------------------------------------------------
// Generic kernel. grid = (ceil(N/128), min(M, 65535)), block = 128.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
k_linear_generic(const int8_t *__restrict__ Xq, int M, int K, int ldq,
                 const float *__restrict__ sx,
                 const uint8_t *__restrict__ Wp, int ldp, const float *__restrict__ sw, int N,
                 const float *__restrict__ bias, unsigned flags, void *__restrict__ Y, int ldy, ZpArgs zpa) {
    griddep_launch_dependents();
    griddep_wait();
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const uint8_t *wr = Wp + (size_t)n * ldp;
    const float swn = ld_dep(sw + n);
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
        const int8_t *xr = Xq + (size_t)m * ldq;
        int32_t acc = 0;
        for (int k = 0; k < K; k += 2) {
            // byte k/2: code k in the low nibble, code k + 1 in the high one
            const uint32_t b = ld_dep_u8(wr + (k >> 1));
            acc += ld_dep_s8(xr + k) * ((int)((b & 0xFu) ^ 8u) - 8);
            if (k + 1 < K) acc += ld_dep_s8(xr + k + 1) * ((int)((b >> 4) ^ 8u) - 8);
        }
        store_out(Y, ldy, m, n, zp_fix(acc, zpa, m, n), ld_dep(sx + m), swn, bias, flags);
    }
}

// ---------------------------------------------------------------------------
// Decode kernels.
//
// Block = 8 warps = one 16-channel row block of the weight matrix; warp w owns
// the 128-k chunks c = w, w+8, w+16, ... of K, so the block's warps read 512
// contiguous bytes of each weight row between them. blockIdx.y selects a tile
// of 8*NTG activation rows (tokens).
//
// mma.sync.m16n8k32 (A 16x32 row-major, B 32x8 col-major, s8 -> s32) with the
// weights as A and the tokens as B. The dot product does not care which
// physical k sits in which of the instruction's 32 k-slots, as long as A and B
// agree. Thread (g = lane/4, t = lane%4) loads 16 bytes of weight rows g and
// g+8 per chunk: bytes [64c + 16t, +16) = k in [128c + 32t, +32). Word j of
// them (k = 128c + 32t + 8j .. +7) feeds MMA j: its low nibbles (even k) go to
// A slots 4t..4t+3 and its high nibbles (odd k) to slots 16+4t..16+4t+3. The
// B fragment of the same thread covers the same slots, so it takes the even
// and odd bytes of xq[token][128c + 32t + 8j .. +7].
//
// Only the first kp = round_up(ceil(K/2), 16) bytes of a packed row are read
// (codes and zero pad nibbles); any row stride past them is never touched.
//
// Programmatic dependent launch. Weights are streamed before
// griddepcontrol.wait only where they are known to be final: behind this
// library's activation pass (which lets a dependent start only after all
// earlier work has completed), or when the caller passes
// W4A8_STATIC_WEIGHTS. Otherwise the block only asks for its weight rows to be
// brought into L2 before the wait, and loads them after it.
// ---------------------------------------------------------------------------
constexpr int DEC_WARPS = 8;
// chunks per warp per batch of loads: 4, so for K <= 4096 a warp's whole
// share of the weights is in registers from before the dependency wait, for
// one token group and for two (the second group's activation fragments take
// the kernel from 90 to about 120 registers, still two blocks per SM; with 2
// chunks per batch the second batch of weight loads left HBM latency after
// the wait)
template <int NTG>
constexpr int dec_unroll() { return 4; }

// Packed bytes of a row that the kernels read: codes plus pad, 16-aligned.
__host__ __device__ __forceinline__ int packed_row_bytes(int K) { return ((K + 1) / 2 + 15) / 16 * 16; }

__device__ __forceinline__ void mma_s8_16832(int32_t (&c)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The weight rows n0 + g and n0 + g + 8 as thread (g, t) of a decode warp
// reads them: one 16-byte piece of each per chunk. Weights are read once per
// call, so the loads are marked streaming (evict-first), which keeps the
// activations and outputs in L2.
template <int UNROLL>
struct DecodeWeights {
    const uint8_t *lo, *hi;
    bool lo_ok, hi_ok;
    int kp, t16;
    __device__ __forceinline__ DecodeWeights(const uint8_t *Wp, int ldp, int N, int n0, int g, int t, int K) {
        lo_ok = n0 + g < N;
        hi_ok = n0 + g + 8 < N;
        t16 = 16 * t;
        lo = Wp + (size_t)(lo_ok ? n0 + g : 0) * ldp + t16;
        hi = Wp + (size_t)(hi_ok ? n0 + g + 8 : 0) * ldp + t16;
        kp = packed_row_bytes(K);
    }
    // chunks cb, cb + DEC_WARPS, ... (pieces past kp read as zeros)
    __device__ __forceinline__ void load(int cb, uint4 (&wa)[UNROLL], uint4 (&wb)[UNROLL]) const {
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int off = 64 * (cb + u * DEC_WARPS);
            const bool in = off + t16 < kp;
            const uint4 z = make_uint4(0, 0, 0, 0);
            wa[u] = (in && lo_ok) ? ld_stream_v4(lo + off) : z;
            wb[u] = (in && hi_ok) ? ld_stream_v4(hi + off) : z;
        }
    }
};

// MMAs of one batch: chunks cb + u * DEC_WARPS (u < UNROLL) that exist.
template <int NTG, int UNROLL>
__device__ __forceinline__ void decode_mma_batch(int32_t (&acc)[NTG][4], const uint4 (&wa)[UNROLL],
                                                 const uint4 (&wb)[UNROLL], const uint4 (&xv)[UNROLL][NTG][2],
                                                 int cb, int nchunks) {
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
        if (cb + u * DEC_WARPS >= nchunks) continue;  // warp-uniform
        const uint32_t pa[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
        const uint32_t pb[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t alo, ahi, blo, bhi;
            unpack_s4x8(pa[j], alo, ahi);
            unpack_s4x8(pb[j], blo, bhi);
#pragma unroll
            for (int i = 0; i < NTG; ++i) {
                const uint4 &v = xv[u][i][j >> 1];
                const uint32_t x0 = (j & 1) ? v.z : v.x;
                const uint32_t x1 = (j & 1) ? v.w : v.y;
                const uint32_t b0 = __byte_perm(x0, x1, 0x6420);  // even k
                const uint32_t b1 = __byte_perm(x0, x1, 0x7531);  // odd k
                mma_s8_16832(acc[i], alo, blo, ahi, bhi, b0, b1);
            }
        }
    }
}

// Sum the warps' C fragments (rows g, g+8 = channels, columns 2t, 2t+1 =
// tokens) through shared memory; returns the block total of output e
// (channel e % 16, token e / 16) for e < 16 * TOK.
template <int NTG>
__device__ __forceinline__ int32_t decode_reduce(int32_t (*red)[16][8 * NTG + 1], const int32_t (&acc)[NTG][4],
                                                 int warp, int g, int t) {
#pragma unroll
    for (int i = 0; i < NTG; ++i) {
        red[warp][g][8 * i + 2 * t] = acc[i][0];
        red[warp][g][8 * i + 2 * t + 1] = acc[i][1];
        red[warp][g + 8][8 * i + 2 * t] = acc[i][2];
        red[warp][g + 8][8 * i + 2 * t + 1] = acc[i][3];
    }
    __syncthreads();
    int32_t s = 0;
    if (threadIdx.x < 16 * 8 * NTG) {
        const int e_ch = threadIdx.x % 16, e_tk = threadIdx.x / 16;
#pragma unroll
        for (int w = 0; w < DEC_WARPS; ++w) s += red[w][e_ch][e_tk];
    }
    return s;
}

// Decode kernel on INT8 activations (from the activation pass or the caller).
// EARLY: the weights are final when the kernel starts (see above).
template <int NTG, bool EARLY>
__global__ void __launch_bounds__(DEC_WARPS * 32, 2)
k_linear_decode(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                const uint8_t *Wp, int ldp, const float *sw, int N,
                const float *bias, unsigned flags, void *Y, int ldy, ZpArgs zpa) {
    constexpr int TOK = 8 * NTG;
    constexpr int UNROLL = dec_unroll<NTG>();
    static_assert(16 * TOK <= DEC_WARPS * 32, "one epilogue element per thread");
    __shared__ int32_t red[DEC_WARPS][16][TOK + 1];
    griddep_launch_dependents();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * TOK;
    const DecodeWeights<UNROLL> W(Wp, ldp, N, n0, g, t, K);
    const int nchunks = (W.kp + 63) / 64;
    uint4 wa[UNROLL], wb[UNROLL];
    if constexpr (EARLY) {
        W.load(warp, wa, wb);
    } else if (threadIdx.x == 0) {
        prefetch_l2_bulk(Wp + (size_t)n0 * ldp, (uint32_t)(min(16, N - n0) * ldp));
    }
    griddep_wait();
    if constexpr (!EARLY) W.load(warp, wa, wb);

    // Epilogue operands, fetched now so their latency hides under the stream:
    // thread e finishes output (channel n0 + e % 16, token m0 + e / 16).
    const int e_ch = threadIdx.x % 16, e_tk = threadIdx.x / 16;
    const bool e_ok = threadIdx.x < 16 * TOK && n0 + e_ch < N && m0 + e_tk < M;
    float e_sw = 1.0f, e_sx = 1.0f;
    if (e_ok) {
        e_sw = ld_dep(sw + n0 + e_ch);
        e_sx = ld_dep(sx + m0 + e_tk);
    }

    int32_t acc[NTG][4];
#pragma unroll
    for (int i = 0; i < NTG; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0;

    for (int cb = warp; cb < nchunks; cb += DEC_WARPS * UNROLL) {
        // Issue every load of this batch before any use: weights (the first
        // batch is already out) and the matching INT8 activations (an
        // out-of-range piece reads as zeros).
        if (cb != warp) W.load(cb, wa, wb);
        uint4 xv[UNROLL][NTG][2];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int kbase = 128 * (cb + u * DEC_WARPS) + 32 * t;
#pragma unroll
            for (int i = 0; i < NTG; ++i) {
                const int m = m0 + 8 * i + g;
                const int8_t *xr = Xq + (size_t)m * ldq + kbase;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const bool ok = m < M && kbase + 16 * h < ldq;
                    xv[u][i][h] = ok ? ld_dep_v4(xr + 16 * h) : make_uint4(0, 0, 0, 0);
                }
            }
        }
        decode_mma_batch<NTG, UNROLL>(acc, wa, wb, xv, cb, nchunks);
    }

    const int32_t s = decode_reduce<NTG>(red, acc, warp, g, t);
    if (e_ok) store_out(Y, ldy, m0 + e_tk, n0 + e_ch, zp_fix(s, zpa, m0 + e_tk, n0 + e_ch), e_sx, e_sw, bias, flags);
}

}  // namespace w4a8
