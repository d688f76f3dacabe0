// W8A8 product kernels on the CUDA cores and the legacy integer tensor path:
// the INT8 path that the Keras guide "INT4 quantization in Keras" (section
// "How it works", closing paragraph) says its INT4 steps extend. Same steps
// 3-6 as the INT4 layer with one INT8 weight code per byte (scale 127 /
// abs-max, codes in [-127, 127]) and no unpack:
//   acc[m][n] = sum_k xq[m][k] * q8[n][k];  y = float(acc) / (sx[m] * sw[n]).
// Wq is [N][ldw8] bytes, K-contiguous per output channel; bytes k in
// [K, round_up(K, 16)) of a row must be 0 (w8_quantize writes them so) and
// bytes past round_up(K, 16) are never read.
#pragma once

#include "common.cuh"
#include "linear_simt.cuh"

namespace w4a8 {

// Bytes of an INT8 weight row that the kernels read: K rounded up to 16.
__host__ __device__ __forceinline__ int w8_row_bytes(int K) { return (K + 15) / 16 * 16; }

// Generic kernel: one thread per (output channel, activation row), any shape.
__global__ void __launch_bounds__(128)
k_linear8_generic(const int8_t *__restrict__ Xq, int M, int K, int ldq, const float *__restrict__ sx,
                  const int8_t *__restrict__ Wq, int ldw8, const float *__restrict__ sw, int N,
                  const float *__restrict__ bias, unsigned flags, void *__restrict__ Y, int ldy) {
    griddep_launch_dependents();
    griddep_wait();
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const int8_t *wr = Wq + (size_t)n * ldw8;
    const float swn = ld_dep(sw + n);
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
        const int8_t *xr = Xq + (size_t)m * ldq;
        int32_t acc = 0;
        for (int k = 0; k < K; ++k) acc += ld_dep_s8(xr + k) * ld_dep_s8(wr + k);
        store_out(Y, ldy, m, n, acc, ld_dep(sx + m), swn, bias, flags);
    }
}

// ---------------------------------------------------------------------------
// Decode kernel (M <= 16 per tile): block = 8 warps = one 16-channel row
// block; warp w owns the 128-k chunks c = w, w + 8, ... Thread (g = lane / 4,
// t = lane % 4) reads the 32 bytes [128c + 32t, +32) of weight rows g and
// g + 8 and of its token rows: word j (k = 128c + 32t + 4j .. +3) of each.
// MMA q of the chunk (mma.sync.m16n8k32, s8 -> s32) takes words 2q and
// 2q + 1: the A slots 4t..4t+3 hold word 2q of rows g / g + 8, slots
// 16+4t..16+4t+3 word 2q + 1, and the B fragment of the same thread the
// same two words of the token row - so A and B agree on every k and the
// 32 slots of the four threads t cover 32 distinct k. No unpack and no byte
// permutes.
//
// Programmatic dependent launch as for the INT4 decode kernel: with final
// weights (behind the activation pass, or W4A8_STATIC_WEIGHTS) the first
// batch of weight loads goes out before griddepcontrol.wait; otherwise the
// block's rows are prefetched into L2 before it.
// ---------------------------------------------------------------------------
constexpr int DEC8_UNROLL = 2;  // chunks per warp per batch: 8 x 16-byte weight loads in flight

struct DecodeWeights8 {
    const int8_t *lo, *hi;
    bool lo_ok, hi_ok;
    int kb, t32;
    __device__ __forceinline__ DecodeWeights8(const int8_t *Wq, int ldw8, int N, int n0, int g, int t, int K) {
        lo_ok = n0 + g < N;
        hi_ok = n0 + g + 8 < N;
        t32 = 32 * t;
        lo = Wq + (size_t)(lo_ok ? n0 + g : 0) * ldw8 + t32;
        hi = Wq + (size_t)(hi_ok ? n0 + g + 8 : 0) * ldw8 + t32;
        kb = w8_row_bytes(K);
    }
    // chunks cb + u * DEC_WARPS; 16-byte pieces at or past kb read as zeros
    __device__ __forceinline__ void load(int cb, uint4 (&wa)[DEC8_UNROLL][2], uint4 (&wb)[DEC8_UNROLL][2]) const {
#pragma unroll
        for (int u = 0; u < DEC8_UNROLL; ++u) {
            const int off = 128 * (cb + u * DEC_WARPS);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool in = off + t32 + 16 * h < kb;
                const uint4 z = make_uint4(0, 0, 0, 0);
                wa[u][h] = (in && lo_ok) ? ld_stream_v4(lo + off + 16 * h) : z;
                wb[u][h] = (in && hi_ok) ? ld_stream_v4(hi + off + 16 * h) : z;
            }
        }
    }
};

template <int NTG, bool EARLY>
__global__ void __launch_bounds__(DEC_WARPS * 32)
k_linear8_decode(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                 const int8_t *Wq, int ldw8, const float *sw, int N,
                 const float *bias, unsigned flags, void *Y, int ldy) {
    constexpr int TOK = 8 * NTG;
    static_assert(16 * TOK <= DEC_WARPS * 32, "one epilogue element per thread");
    __shared__ int32_t red[DEC_WARPS][16][TOK + 1];
    griddep_launch_dependents();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * TOK;
    const DecodeWeights8 W(Wq, ldw8, N, n0, g, t, K);
    const int nchunks = (W.kb + 127) / 128;
    uint4 wa[DEC8_UNROLL][2], wb[DEC8_UNROLL][2];
    if constexpr (EARLY) {
        W.load(warp, wa, wb);
    } else if (threadIdx.x == 0) {
        prefetch_l2_bulk(Wq + (size_t)n0 * ldw8, (uint32_t)(min(16, N - n0) * ldw8));
    }
    griddep_wait();
    if constexpr (!EARLY) W.load(warp, wa, wb);

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

    for (int cb = warp; cb < nchunks; cb += DEC_WARPS * DEC8_UNROLL) {
        if (cb != warp) W.load(cb, wa, wb);
        uint4 xv[DEC8_UNROLL][NTG][2];
#pragma unroll
        for (int u = 0; u < DEC8_UNROLL; ++u) {
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
#pragma unroll
        for (int u = 0; u < DEC8_UNROLL; ++u) {
            if (cb + u * DEC_WARPS >= nchunks) continue;  // warp-uniform
            const uint32_t a[8] = {wa[u][0].x, wa[u][0].y, wa[u][0].z, wa[u][0].w,
                                   wa[u][1].x, wa[u][1].y, wa[u][1].z, wa[u][1].w};
            const uint32_t b[8] = {wb[u][0].x, wb[u][0].y, wb[u][0].z, wb[u][0].w,
                                   wb[u][1].x, wb[u][1].y, wb[u][1].z, wb[u][1].w};
#pragma unroll
            for (int i = 0; i < NTG; ++i) {
                const uint32_t x[8] = {xv[u][i][0].x, xv[u][i][0].y, xv[u][i][0].z, xv[u][i][0].w,
                                       xv[u][i][1].x, xv[u][i][1].y, xv[u][i][1].z, xv[u][i][1].w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    mma_s8_16832(acc[i], a[2 * q], b[2 * q], a[2 * q + 1], b[2 * q + 1], x[2 * q], x[2 * q + 1]);
            }
        }
    }

    const int32_t s = decode_reduce<NTG>(red, acc, warp, g, t);
    if (e_ok) store_out(Y, ldy, m0 + e_tk, n0 + e_ch, s, e_sx, e_sw, bias, flags);
}

}  // namespace w4a8
