// Asymmetric INT4 weights with a per-output-channel zero point (the uniform
// asymmetric quantization of the "INT4" concept page, section 4.1, and the
// formulas of the "4-bit Integer Quantization for LLMs" page, section "Weight
// quantization"), with the W4A8 layer's INT8 activations:
//   sa[n] = 15 / (max_k W[k][n] - min_k W[k][n])   (1 when they are equal)
//   zp[n] = -rne(min_k W[k][n] * sa[n])             (an integer)
//   q     = clamp(rne(w * sa[n]) + zp[n], 0, 15)
//   acc   = sum_k xq[m][k] * (q - zp[n]);  y = float(acc) / (sx[m] * sa[n])
// Storage: each code is kept as the signed nibble q - 8 (two's complement,
// i.e. q XOR 8), pad nibbles 0, in the W4A8 packed layout. The W4A8 product
// kernels then compute acc' = sum_k xq * (q - 8) unchanged, and
//   acc = acc' - (zp - 8) * rowsum,  rowsum[m] = sum_k xq[m][k],
// which the product kernels apply in their epilogues (ZpArgs in common.cuh;
// 64-bit, then the same float32 operations as every other path). The row sums
// come from the activation pass, or from k_row_sum8 for INT8 input.
#pragma once

#include <climits>

#include "common.cuh"

namespace w4a8 {
namespace zpt {

// Float order as signed-int order (finite values): non-negative floats keep
// their bits, negative ones flip their magnitude bits.
__device__ __forceinline__ int order_key(float f) {
    const int b = __float_as_int(f);
    return b >= 0 ? b : b ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float from_order_key(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7FFFFFFF); }

// min keys start at INT_MAX, max keys at INT_MIN.
__global__ void k_minmax_init(int *__restrict__ lo_key, int *__restrict__ hi_key, int N) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n < N) {
        lo_key[n] = INT_MAX;
        hi_key[n] = INT_MIN;
    }
}

// Column min and max of W [K][ldw] over a K-slice per blockIdx.y; warp w
// walks rows k0 + w, + 8, ... (row-coalesced), the block's 8 warps meet in
// shared memory, the K-slices in the two key arrays through atomics.
// grid = (ceil(N / 32), k_splits), block = 256.
__global__ void __launch_bounds__(256)
k_col_minmax(const float *__restrict__ W, int K, int N, int ldw, int rows_per_split, int *__restrict__ lo_key,
             int *__restrict__ hi_key) {
    __shared__ float rlo[8][33], rhi[8][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * 32 + lane;
    const int k0 = blockIdx.y * rows_per_split;
    const int k1 = min(K, k0 + rows_per_split);
    float lo = INFINITY, hi = -INFINITY;
    if (n < N)
        for (int k = k0 + warp; k < k1; k += 8) {
            const float v = __ldg(W + (size_t)k * ldw + n);
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
        }
    rlo[warp][lane] = lo;
    rhi[warp][lane] = hi;
    __syncthreads();
    if (warp == 0 && n < N) {
        for (int i = 1; i < 8; ++i) {
            lo = fminf(lo, rlo[i][lane]);
            hi = fmaxf(hi, rhi[i][lane]);
        }
        if (k0 < k1) {
            atomicMin(lo_key + n, order_key(lo));
            atomicMax(hi_key + n, order_key(hi));
        }
    }
}

// Keys -> sa (in place over hi_key) and zp (in place over lo_key).
__global__ void k_zp_finalize(int *__restrict__ lo_key, int *__restrict__ hi_key, int N) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const float lo = from_order_key(lo_key[n]), hi = from_order_key(hi_key[n]);
    const float range = __fsub_rn(hi, lo);
    const float sa = range == 0.0f ? 1.0f : __fdiv_rn(15.0f, range);
    reinterpret_cast<float *>(hi_key)[n] = sa;
    lo_key[n] = -__float2int_rn(__fmul_rn(lo, sa));
}

// Codes, stored as q - 8: a tile of 64 k x 32 channels; warp w reads rows
// k0 + 8w .. + 7 of its lane's channel and packs the 8 codes into one 32-bit
// word (code k0 + 8w + i in bits 4i..4i+3); the words leave through shared
// memory as 16-byte row stores, every byte of [0, ldp) written.
// grid = (ceil(N / 32), ceil(2 * ldp / 64)), block = 256.
__global__ void __launch_bounds__(256)
k_quant_pack_z(const float *__restrict__ W, int K, int N, int ldw, const float *__restrict__ sa,
               const int *__restrict__ zp, uint8_t *__restrict__ Wp, int ldp) {
    __shared__ __align__(16) uint32_t pk[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * 32 + lane;
    const int k0 = blockIdx.y * 64 + 8 * warp;
    const float s = n < N ? __ldg(sa + n) : 1.0f;
    const int z = n < N ? __ldg(zp + n) : 0;
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int k = k0 + i;
        if (k < K && n < N) {
            const float v = __ldg(W + (size_t)k * ldw + n);
            const int q = clampi(__float2int_rn(__fmul_rn(v, s)) + z, 0, 15);
            word |= ((uint32_t)(q - 8) & 0xFu) << (4 * i);
        }
    }
    pk[warp][lane] = word;
    __syncthreads();
    if (threadIdx.x < 64) {
        const int r = threadIdx.x % 32, h = threadIdx.x / 32;
        const int nn = blockIdx.x * 32 + r;
        const int byte0 = blockIdx.y * 32 + 16 * h;
        if (nn < N && byte0 < ldp)
            *reinterpret_cast<uint4 *>(Wp + (size_t)nn * ldp + byte0) =
                make_uint4(pk[4 * h][r], pk[4 * h + 1][r], pk[4 * h + 2][r], pk[4 * h + 3][r]);
    }
}

// rowsum[m] = sum_{k < K} xq[m][k] (bytes past K are not counted). One block
// of 256 threads per row, grid-stride over rows.
__global__ void __launch_bounds__(256)
k_row_sum8(const int8_t *Xq, int M, int K, int ldq, int *rowsum) {
    __shared__ int part[8];
    // wait first: a dependent that starts after this point knows that all
    // earlier work on the stream has finished (it may then fetch final
    // weights before its own wait, as behind the activation pass)
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const int8_t *row = Xq + (size_t)m * ldq;
        int s = 0;
        for (int c = threadIdx.x; 16 * c < K; c += 256) {
            const uint4 v = ld_dep_v4(row + 16 * c);
            if (16 * c + 16 <= K) {
                s = __dp4a((int)v.x, 0x01010101, s);
                s = __dp4a((int)v.y, 0x01010101, s);
                s = __dp4a((int)v.z, 0x01010101, s);
                s = __dp4a((int)v.w, 0x01010101, s);
            } else {
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                for (int b = 0; 16 * c + b < K; ++b) s += (int)(int8_t)((w[b >> 2] >> (8 * (b & 3))) & 0xFFu);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) part[warp] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            int t = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) t += part[w];
            rowsum[m] = t;
        }
        __syncthreads();
    }
}

}  // namespace zpt
}  // namespace w4a8
