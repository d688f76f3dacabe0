// Weight quantize+pack and activation quantize kernels.
//
// Weights (Keras guide "INT4 quantization in Keras", "How it works", steps 1-2):
//   sw[n] = 7 / max_k |W[k][n]| (1 for an all-zero column);
//   q = clamp(rne(W[k][n] * sw[n]), -8, 7), packed two per byte along K.
// Activations (step 3): sx[m] = 127 / max_k |X[m][k]| (1 for an all-zero row);
//   xq = clamp(rne(X[m][k] * sx[m]), -127, 127).
#pragma once

#include "common.cuh"

namespace w4a8 {

// ---------------------------------------------------------------------------
// Weight pass 1: column abs-max. W is [K][ldw] (columns = output channels), so
// a warp reads 32 consecutive columns of one row (128 contiguous bytes) and
// the block's 8 warps walk disjoint rows of a K-slice. The per-column maxima
// of all K-slices meet in amax_bits[n] through an integer atomicMax on the
// float bit patterns (valid because every value is >= +0).
// grid = (ceil(N/32), k_splits), block = (32, 8).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_col_absmax(const float *__restrict__ W, int K, int N, int ldw, int rows_per_split,
             unsigned *__restrict__ amax_bits) {
    __shared__ float red[8][33];
    const int n = blockIdx.x * 32 + threadIdx.x;
    const int k0 = blockIdx.y * rows_per_split;
    const int k1 = min(K, k0 + rows_per_split);
    float m0 = 0.f, m1 = 0.f, m2 = 0.f, m3 = 0.f;
    if (n < N) {
        const float *col = W + n;
        int k = k0 + threadIdx.y;
        for (; k + 24 < k1; k += 32) {
            m0 = fmaxf(m0, fabsf(__ldg(col + (size_t)k * ldw)));
            m1 = fmaxf(m1, fabsf(__ldg(col + (size_t)(k + 8) * ldw)));
            m2 = fmaxf(m2, fabsf(__ldg(col + (size_t)(k + 16) * ldw)));
            m3 = fmaxf(m3, fabsf(__ldg(col + (size_t)(k + 24) * ldw)));
        }
        for (; k < k1; k += 8) m0 = fmaxf(m0, fabsf(__ldg(col + (size_t)k * ldw)));
    }
    red[threadIdx.y][threadIdx.x] = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
    __syncthreads();
    if (threadIdx.y == 0 && n < N) {
        float m = red[0][threadIdx.x];
#pragma unroll
        for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i][threadIdx.x]);
        atomicMax(&amax_bits[n], __float_as_uint(m));
    }
}

__device__ __forceinline__ float weight_scale_from_amax(unsigned bits) {
    float a = __uint_as_float(bits);
    return a == 0.0f ? 1.0f : __fdiv_rn(7.0f, a);
}

// ---------------------------------------------------------------------------
// Weight pass 2: quantize and pack a tile of 64 k x 32 output channels.
// Reads are row-coalesced (a warp reads 32 columns of one row); the codes are
// transposed through shared memory so each output channel's 32 bytes of
// packed nibbles leave as two 16-byte stores. Tiles cover k in [0, 2*ldp), so
// every byte of every packed row (pad bytes included) is written.
// grid = (ceil(N/32), ceil(2*ldp/64)), block = (32, 8).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_quant_pack(const float *__restrict__ W, int K, int N, int ldw,
             const unsigned *__restrict__ amax_bits, uint8_t *__restrict__ Wp, int ldp) {
    __shared__ int8_t qs[32][64 + 4];
    const int n = blockIdx.x * 32 + threadIdx.x;
    const int k0 = blockIdx.y * 64;
    float s = 1.0f;
    if (n < N) s = weight_scale_from_amax(__ldg(amax_bits + n));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int kk = threadIdx.y + 8 * i;
        const int k = k0 + kk;
        int q = 0;
        if (n < N && k < K) {
            float t = __fmul_rn(__ldg(W + (size_t)k * ldw + n), s);
            q = clampi(__float2int_rn(t), -8, 7);
        }
        qs[threadIdx.x][kk] = (int8_t)q;
    }
    __syncthreads();
    const int t = threadIdx.y * 32 + threadIdx.x;
    if (t < 64) {
        const int r = t >> 1, h = t & 1;
        const int nn = blockIdx.x * 32 + r;
        const int byte0 = k0 / 2 + 16 * h;  // a multiple of 16, as is ldp
        if (nn < N && byte0 < ldp) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t v = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int kk = 32 * h + 8 * j + 2 * b;
                    uint32_t lo = (uint32_t)(uint8_t)qs[r][kk] & 0xFu;
                    uint32_t hi = (uint32_t)(uint8_t)qs[r][kk + 1] & 0xFu;
                    v |= (lo | (hi << 4)) << (8 * b);
                }
                w[j] = v;
            }
            *reinterpret_cast<uint4 *>(Wp + (size_t)nn * ldp + byte0) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// Weight pass 3: turn the abs-max bits into the scale, in place.
__global__ void k_weight_scale_finalize(float *__restrict__ sw, int N) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n < N) {
        unsigned bits = reinterpret_cast<unsigned *>(sw)[n];
        sw[n] = weight_scale_from_amax(bits);
    }
}

// ---------------------------------------------------------------------------
// Activation quantization: one block per row (grid-stride over rows).
// The row is read once into registers (VPT floats per thread; longer rows
// are re-read for the quantization pass), its abs-max reduced with warp
// shuffles and then across warps, and the codes leave 4 per 32-bit store.
// Bytes K..ldq-1 of each row are written 0.
// ---------------------------------------------------------------------------
template <int THREADS, int VPT>
__global__ void __launch_bounds__(THREADS)
k_act_quant(const float *__restrict__ X, int M, int K, int ldx,
            int8_t *__restrict__ Xq, int ldq, float *__restrict__ sx, int vec4) {
    static_assert(THREADS % 32 == 0 && THREADS <= 1024 && VPT % 4 == 0, "block shape");
    __shared__ float red[THREADS / 32];
    // Let the next kernel launch now: it only prefetches weights before its
    // own griddepcontrol.wait, which returns after this grid has finished.
    // Every block triggers at entry, so all of this grid is resident before
    // any dependent block can take an SM slot.
    griddep_launch_dependents();
    griddep_wait();  // X may be written by the previous kernel
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // Thread j of the block owns the 4-element groups j, j + THREADS, ...
    constexpr int G = VPT / 4;
    const bool in_regs = K <= THREADS * VPT;
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const float *x = X + (size_t)m * ldx;
        float v[G][4];
        float amax = 0.0f;
        if (in_regs) {
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
                const int k = 4 * (threadIdx.x + gi * THREADS);
                if (vec4 && k + 3 < K) {
                    const float4 f = __ldg(reinterpret_cast<const float4 *>(x + k));
                    v[gi][0] = f.x; v[gi][1] = f.y; v[gi][2] = f.z; v[gi][3] = f.w;
                } else {
#pragma unroll
                    for (int b = 0; b < 4; ++b) v[gi][b] = (k + b < K) ? __ldg(x + k + b) : 0.0f;
                }
#pragma unroll
                for (int b = 0; b < 4; ++b) amax = fmaxf(amax, fabsf(v[gi][b]));
            }
        } else {
            for (int k = threadIdx.x; k < K; k += THREADS) amax = fmaxf(amax, fabsf(__ldg(x + k)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        float a = red[0];
#pragma unroll
        for (int i = 1; i < THREADS / 32; ++i) a = fmaxf(a, red[i]);
        const float s = a == 0.0f ? 1.0f : __fdiv_rn(127.0f, a);
        if (threadIdx.x == 0) sx[m] = s;
        uint32_t *q4 = reinterpret_cast<uint32_t *>(Xq + (size_t)m * ldq);
        if (in_regs) {
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
                const int j = threadIdx.x + gi * THREADS;
                if (4 * j < ldq) {
                    uint32_t packed = 0;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int q = (4 * j + b < K) ? clampi(__float2int_rn(__fmul_rn(v[gi][b], s)), -127, 127) : 0;
                        packed |= (uint32_t)(q & 0xFF) << (8 * b);
                    }
                    q4[j] = packed;
                }
            }
            for (int j = threadIdx.x + G * THREADS; j < ldq / 4; j += THREADS) q4[j] = 0;
        } else {
            for (int j = threadIdx.x; j < ldq / 4; j += THREADS) {
                uint32_t packed = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int k = 4 * j + b;
                    const int q = (k < K) ? clampi(__float2int_rn(__fmul_rn(__ldg(x + k), s)), -127, 127) : 0;
                    packed |= (uint32_t)(q & 0xFF) << (8 * b);
                }
                q4[j] = packed;
            }
        }
        __syncthreads();  // red is reused by the next row
    }
}

}  // namespace w4a8
