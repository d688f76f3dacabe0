// Group-wise INT4 weights ("INT4" concept page, section 4.2, group
// quantization: every group of group_size = 128 weights along the input axis
// has its own scale and zero point) with the W4A8 layer's INT8 activations:
//   per (output channel n, group g = k / 128): sa[n][g] = 15 / (max - min)
//   (1 when equal), zp[n][g] = -rne(min * sa), q = clamp(rne(w * sa) + zp, 0, 15);
//   y = sum_g float(acc_g) / (sx * sa[n][g]),  acc_g = sum_{k in g} xq * (q - zp).
// Storage: the packed layout of the zero-point form (signed nibbles q - 8,
// pad 0); one group is exactly one 64-byte chunk of a packed row, so the
// decode kernel's chunk loop is the group loop.
#pragma once

#include "common.cuh"
#include "linear_simt.cuh"

namespace w4a8 {
namespace grp {

constexpr int G = 128;  // weights per group along K

__host__ __device__ __forceinline__ int groups_of(int K) { return (K + G - 1) / G; }

// Quantize and pack one (channel, group) per thread: the group's min and
// max, its scale and zero point, then its 64 packed bytes (four 16-byte
// stores, clipped to the row's ldp bytes). grid = (ceil(N / 128), ng),
// block = 128: adjacent threads take adjacent channels (coalesced rows of W).
__global__ void __launch_bounds__(128)
k_quant_pack_g(const float *__restrict__ W, int K, int N, int ldw, uint8_t *__restrict__ Wp, int ldp,
               float *__restrict__ sa, int32_t *__restrict__ zp, int ng) {
    const int n = blockIdx.x * 128 + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= N) return;
    const int k0 = g * G, k1 = min(K, k0 + G);
    float lo = __ldg(W + (size_t)k0 * ldw + n), hi = lo;
    for (int k = k0 + 1; k < k1; ++k) {
        const float w = __ldg(W + (size_t)k * ldw + n);
        lo = w < lo ? w : lo;
        hi = w > hi ? w : hi;
    }
    const float range = __fsub_rn(hi, lo);
    const float s = range == 0.0f ? 1.0f : __fdiv_rn(15.0f, range);
    const int z = -__float2int_rn(__fmul_rn(lo, s));
    sa[(size_t)n * ng + g] = s;
    zp[(size_t)n * ng + g] = z;
    uint32_t words[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) words[j] = 0;
#pragma unroll
    for (int i = 0; i < G; ++i) {
        const int k = k0 + i;
        if (k < K) {
            const int q = clampi(__float2int_rn(__fmul_rn(__ldg(W + (size_t)k * ldw + n), s)) + z, 0, 15);
            words[i / 8] |= ((uint32_t)(q - 8) & 0xFu) << (4 * (i % 8));
        }
    }
    uint8_t *row = Wp + (size_t)n * ldp;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int byte0 = 64 * g + 16 * j;  // a multiple of 16, as is ldp
        if (byte0 < ldp)
            *reinterpret_cast<uint4 *>(row + byte0) =
                make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
    }
}

// The product, for any M (tiles of 8 * NTG tokens on grid.y). Block = 8 warps
// = one 16-channel row block; warp w takes groups (= chunks) w, w + 8, ...
// exactly as k_linear_decode takes chunks. Per group, the 4 MMAs of the chunk
// go into a fresh INT32 fragment; the token rows' sums over the group (the
// quad of threads that share a token row covers its 128 k) give the
// zero-point correction acc_g = acc' - (zp - 8) * rowsum_g in 64-bit; the
// group's term float(acc_g) / (sx * sa) (the float32 operations of the
// statement) is added to a float32 fragment. The 8 warps' fragments meet in
// shared memory and are summed in warp order; bias, ReLU and the output
// format follow.
template <int NTG, bool EARLY>
__global__ void __launch_bounds__(DEC_WARPS * 32)
k_linear_g(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
           const float *sa, const int32_t *zp, int ng, int N, const float *bias, unsigned flags, void *Y, int ldy) {
    constexpr int TOK = 8 * NTG;
    constexpr int UNROLL = 4;
    static_assert(16 * TOK <= DEC_WARPS * 32, "one epilogue element per thread");
    __shared__ float red[DEC_WARPS][16][TOK + 1];
    griddep_launch_dependents();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * TOK;
    const DecodeWeights<UNROLL> Wt(Wp, ldp, N, n0, g, t, K);
    const int nchunks = (Wt.kp + 63) / 64;  // = ng
    uint4 wa[UNROLL], wb[UNROLL];
    if constexpr (EARLY) {
        Wt.load(warp, wa, wb);
    } else if (threadIdx.x == 0) {
        prefetch_l2_bulk(Wp + (size_t)n0 * ldp, (uint32_t)(min(16, N - n0) * ldp));
    }
    griddep_wait();
    if constexpr (!EARLY) Wt.load(warp, wa, wb);

    // this thread's C columns are tokens m0 + 8i + 2t and + 1
    float sxc[NTG][2];
#pragma unroll
    for (int i = 0; i < NTG; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = m0 + 8 * i + 2 * t + h;
            sxc[i][h] = m < M ? ld_dep(sx + m) : 1.0f;
        }
    const bool lo_ok = n0 + g < N, hi_ok = n0 + g + 8 < N;
    float yf[NTG][4];
#pragma unroll
    for (int i = 0; i < NTG; ++i) yf[i][0] = yf[i][1] = yf[i][2] = yf[i][3] = 0.0f;

    for (int cb = warp; cb < nchunks; cb += DEC_WARPS * UNROLL) {
        if (cb != warp) Wt.load(cb, wa, wb);
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
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int c = cb + u * DEC_WARPS;
            if (c >= nchunks) continue;  // warp-uniform
            // the group's scale and zero point of this thread's two channels
            const float s_lo = lo_ok ? ld_dep(sa + (size_t)(n0 + g) * ng + c) : 1.0f;
            const float s_hi = hi_ok ? ld_dep(sa + (size_t)(n0 + g + 8) * ng + c) : 1.0f;
            const long long z_lo = lo_ok ? (long long)ld_dep_s32(zp + (size_t)(n0 + g) * ng + c) - 8 : 0;
            const long long z_hi = hi_ok ? (long long)ld_dep_s32(zp + (size_t)(n0 + g + 8) * ng + c) - 8 : 0;
            int32_t acc[NTG][4];
#pragma unroll
            for (int i = 0; i < NTG; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0;
            const uint4 one_a[1] = {wa[u]}, one_b[1] = {wb[u]};
            uint4 one_x[1][NTG][2];
#pragma unroll
            for (int i = 0; i < NTG; ++i) {
                one_x[0][i][0] = xv[u][i][0];
                one_x[0][i][1] = xv[u][i][1];
            }
            decode_mma_batch<NTG, 1>(acc, one_a, one_b, one_x, c, nchunks);
            // token-row sums over the group: this thread's 32 bytes (bytes at
            // k >= K masked off), then the quad of its token row
            const int kb = 128 * c + 32 * t;
            int rs_col[NTG][2];
#pragma unroll
            for (int i = 0; i < NTG; ++i) {
                const uint32_t w8[8] = {xv[u][i][0].x, xv[u][i][0].y, xv[u][i][0].z, xv[u][i][0].w,
                                        xv[u][i][1].x, xv[u][i][1].y, xv[u][i][1].z, xv[u][i][1].w};
                int rs = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int kw = kb + 4 * j;  // k of byte 0 of word j
                    uint32_t v = w8[j];
                    if (kw + 4 > K) v = kw >= K ? 0u : (v & (0xFFFFFFFFu >> (8 * (kw + 4 - K))));
                    rs = __dp4a((int)v, 0x01010101, rs);
                }
                rs += __shfl_xor_sync(0xffffffffu, rs, 1);
                rs += __shfl_xor_sync(0xffffffffu, rs, 2);
                // token column 2t + h lives in the quad of lanes 4 (2t + h) ..
                rs_col[i][0] = __shfl_sync(0xffffffffu, rs, 4 * (2 * t));
                rs_col[i][1] = __shfl_sync(0xffffffffu, rs, 4 * (2 * t + 1));
            }
#pragma unroll
            for (int i = 0; i < NTG; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int h = e & 1;
                    const long long z = e < 2 ? z_lo : z_hi;
                    const float s = e < 2 ? s_lo : s_hi;
                    const long long a = (long long)acc[i][e] - z * (long long)rs_col[i][h];
                    const float term = __fdiv_rn(__int2float_rn((int32_t)a), __fmul_rn(sxc[i][h], s));
                    yf[i][e] = __fadd_rn(yf[i][e], term);
                }
        }
    }

#pragma unroll
    for (int i = 0; i < NTG; ++i) {
        red[warp][g][8 * i + 2 * t] = yf[i][0];
        red[warp][g][8 * i + 2 * t + 1] = yf[i][1];
        red[warp][g + 8][8 * i + 2 * t] = yf[i][2];
        red[warp][g + 8][8 * i + 2 * t + 1] = yf[i][3];
    }
    __syncthreads();
    if (threadIdx.x < 16 * TOK) {
        const int e_ch = threadIdx.x % 16, e_tk = threadIdx.x / 16;
        const int n = n0 + e_ch, m = m0 + e_tk;
        if (n < N && m < M) {
            float y = 0.0f;
#pragma unroll
            for (int w = 0; w < DEC_WARPS; ++w) y = __fadd_rn(y, red[w][e_ch][e_tk]);
            if (bias) y = __fadd_rn(y, ld_dep(bias + n));
            if (flags & W4A8_RELU) y = y > 0.0f ? y : 0.0f;
            const size_t off = (size_t)m * (size_t)ldy + (size_t)n;
            if ((flags & W4A8_OUT_MASK) == W4A8_OUT_BF16)
                static_cast<__nv_bfloat16 *>(Y)[off] = __float2bfloat16_rn(y);
            else
                static_cast<float *>(Y)[off] = y;
        }
    }
}

}  // namespace grp
}  // namespace w4a8
