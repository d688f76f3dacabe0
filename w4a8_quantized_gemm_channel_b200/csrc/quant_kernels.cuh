// Weight quantize+pack and activation quantize kernels.
//
// Weights (Keras guide "INT4 quantization in Keras", "How it works", steps 1-2):
//   sw[n] = 7 / max_k |W[k][n]| (1 for an all-zero column);
//   q = clamp(rne(W[k][n] * sw[n]), -8, 7), packed two per byte along K.
// Activations (step 3): sx[m] = 127 / max_k |X[m][k]| (1 for an all-zero row);
//   xq = clamp(rne(X[m][k] * sx[m]), -127, 127).
// The weight kernels are launched without a programmatic dependency: each
// starts after all earlier work has finished, so its inputs stay constant
// while it runs and are read on the read-only path. The activation kernel is
// a programmatic dependent and reads X with the ld_dep loads.
#pragma once

#include "common.cuh"

namespace w4a8 {

// ---------------------------------------------------------------------------
// Weight pass 1: column abs-max. W is [K][ldw] (columns = output channels).
// VEC = 4: a warp reads 128 consecutive columns of one row as float4 (512
// contiguous bytes); VEC = 1 is the scalar form for unaligned layouts. The
// block's 8 warps walk disjoint rows of a K-slice, 4 rows in flight each;
// the per-column maxima of all K-slices meet in amax_bits[n] through an
// integer atomicMax on the float bit patterns (valid: every value >= +0).
// grid = (ceil(N / (32 * VEC)), k_splits), block = 256.
// ---------------------------------------------------------------------------
template <int VEC>
__global__ void __launch_bounds__(256)
k_col_absmax(const float *__restrict__ W, int K, int N, int ldw, int rows_per_split,
             unsigned *__restrict__ amax_bits) {
    __shared__ float red[8][32 * VEC + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = (blockIdx.x * 32 + lane) * VEC;
    const int k0 = blockIdx.y * rows_per_split;
    const int k1 = min(K, k0 + rows_per_split);
    float m[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) m[c] = 0.0f;
    auto take = [&](const float *p) {
        if constexpr (VEC == 4) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
            m[0] = fmaxf(m[0], fabsf(v.x)); m[1] = fmaxf(m[1], fabsf(v.y));
            m[2] = fmaxf(m[2], fabsf(v.z)); m[3] = fmaxf(m[3], fabsf(v.w));
        } else {
            m[0] = fmaxf(m[0], fabsf(__ldg(p)));
        }
    };
    if (n < N) {
        const float *col = W + n;
        int k = k0 + warp;
        for (; k + 24 < k1; k += 32) {
            take(col + (size_t)k * ldw);
            take(col + (size_t)(k + 8) * ldw);
            take(col + (size_t)(k + 16) * ldw);
            take(col + (size_t)(k + 24) * ldw);
        }
        for (; k < k1; k += 8) take(col + (size_t)k * ldw);
    }
#pragma unroll
    for (int c = 0; c < VEC; ++c) red[warp][lane * VEC + c] = m[c];
    __syncthreads();
    for (int c = threadIdx.x; c < 32 * VEC; c += 256) {
        const int nn = blockIdx.x * 32 * VEC + c;
        if (nn < N) {
            float a = red[0][c];
#pragma unroll
            for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i][c]);
            atomicMax(&amax_bits[nn], __float_as_uint(a));
        }
    }
}

// sw = QMAX / abs-max (1 for an all-zero column): QMAX = 7 for the INT4
// codes, 127 for the INT8 codes of the W8A8 path.
template <int QMAX = 7>
__device__ __forceinline__ float weight_scale_from_amax(unsigned bits) {
    float a = __uint_as_float(bits);
    return a == 0.0f ? 1.0f : __fdiv_rn((float)QMAX, a);
}

// ---------------------------------------------------------------------------
// Weight pass 2: quantize and pack a tile of 64 k x (32 * VEC) output
// channels. Warp w reads the 8 consecutive rows k0 + 8w .. k0 + 8w + 7
// (row-coalesced, float4 per lane for VEC = 4), so each thread holds 8
// consecutive codes of each of its channels and packs them into one 32-bit
// word in registers (code k0 + 8w + i in bits 4i..4i+3: even k in the low
// nibble of its byte). The words go through shared memory as [warp][channel]
// rows (16-byte stores, no bank conflicts); then each channel's four words
// of one half-tile (32 codes) leave as one 16-byte store. Tiles cover k in
// [0, 2*ldp), so every byte of every packed row (pad bytes included) is
// written. grid = (ceil(N / (32 * VEC)), ceil(2*ldp / 64)), block = 256.
// ---------------------------------------------------------------------------
template <int VEC>
__global__ void __launch_bounds__(256)
k_quant_pack(const float *__restrict__ W, int K, int N, int ldw,
             const unsigned *__restrict__ amax_bits, uint8_t *__restrict__ Wp, int ldp) {
    constexpr int COLS = 32 * VEC;
    __shared__ __align__(16) uint32_t pk[8][COLS];  // [warp][channel]: 8 codes of 8 consecutive k
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = blockIdx.x * COLS;
    const int n = nb + lane * VEC;
    const int k0 = blockIdx.y * 64 + 8 * warp;
    float s[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) s[c] = (n + c < N) ? weight_scale_from_amax(__ldg(amax_bits + n + c)) : 1.0f;
    // all eight rows of this thread in flight before any of them is used
    float v[8][VEC];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int k = k0 + i;
        if (k < K && n < N) {
            if constexpr (VEC == 4) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(W + (size_t)k * ldw + n));
                v[i][0] = f.x; v[i][1] = f.y; v[i][2] = f.z; v[i][3] = f.w;
            } else {
                v[i][0] = __ldg(W + (size_t)k * ldw + n);
            }
        } else {
#pragma unroll
            for (int c = 0; c < VEC; ++c) v[i][c] = 0.0f;
        }
    }
    uint32_t word[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
        word[c] = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int q = clampi(__float2int_rn(__fmul_rn(v[i][c], s[c])), -8, 7);
            word[c] |= ((uint32_t)q & 0xFu) << (4 * i);
        }
    }
    if constexpr (VEC == 4)
        *reinterpret_cast<uint4 *>(&pk[warp][lane * 4]) = make_uint4(word[0], word[1], word[2], word[3]);
    else
        pk[warp][lane] = word[0];
    __syncthreads();
    // thread (h, r): channel nb + r, half-tile h = k in [32h, 32h + 32) = the
    // words of warps 4h .. 4h + 3 = 16 packed bytes at byte k_tile/2 + 16h
    for (int tt = threadIdx.x; tt < 2 * COLS; tt += 256) {
        const int r = tt % COLS, h = tt / COLS;
        const int nn = nb + r;
        const int byte0 = blockIdx.y * 32 + 16 * h;  // a multiple of 16, as is ldp
        if (nn < N && byte0 < ldp)
            *reinterpret_cast<uint4 *>(Wp + (size_t)nn * ldp + byte0) =
                make_uint4(pk[4 * h][r], pk[4 * h + 1][r], pk[4 * h + 2][r], pk[4 * h + 3][r]);
    }
}

// ---------------------------------------------------------------------------
// W8A8 weight pass 2 (the INT8 path the guide's INT4 steps extend): codes
// q = clamp(rne(W[k][n] * sw[n]), -127, 127) with sw = 127 / abs-max, one
// byte each, rows Wq[n][0, ldw8) with zero pad. A tile is 32 k x (32 * VEC)
// channels: warp w reads the 4 consecutive rows k0 + 4w .. k0 + 4w + 3
// (row-coalesced), so each thread holds 4 consecutive codes of each of its
// channels as one 32-bit word (code k0 + 4w + i in byte i). The words meet
// in shared memory as [warp][channel] rows; each channel's 8 words (32 k)
// leave as two 16-byte stores. grid = (ceil(N / (32 * VEC)), ceil(ldw8 / 32)),
// block = 256.
// ---------------------------------------------------------------------------
template <int VEC>
__global__ void __launch_bounds__(256)
k_quant8(const float *__restrict__ W, int K, int N, int ldw, const unsigned *__restrict__ amax_bits,
         int8_t *__restrict__ Wq, int ldw8) {
    constexpr int COLS = 32 * VEC;
    __shared__ __align__(16) uint32_t pk[8][COLS];  // [warp][channel]: 4 codes of 4 consecutive k
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = blockIdx.x * COLS;
    const int n = nb + lane * VEC;
    const int k0 = blockIdx.y * 32 + 4 * warp;
    float s[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c)
        s[c] = (n + c < N) ? weight_scale_from_amax<127>(__ldg(amax_bits + n + c)) : 1.0f;
    float v[4][VEC];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int k = k0 + i;
        if (k < K && n < N) {
            if constexpr (VEC == 4) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(W + (size_t)k * ldw + n));
                v[i][0] = f.x; v[i][1] = f.y; v[i][2] = f.z; v[i][3] = f.w;
            } else {
                v[i][0] = __ldg(W + (size_t)k * ldw + n);
            }
        } else {
#pragma unroll
            for (int c = 0; c < VEC; ++c) v[i][c] = 0.0f;
        }
    }
    uint32_t word[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
        word[c] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int q = clampi(__float2int_rn(__fmul_rn(v[i][c], s[c])), -127, 127);
            word[c] |= ((uint32_t)q & 0xFFu) << (8 * i);
        }
    }
    if constexpr (VEC == 4)
        *reinterpret_cast<uint4 *>(&pk[warp][lane * 4]) = make_uint4(word[0], word[1], word[2], word[3]);
    else
        pk[warp][lane] = word[0];
    __syncthreads();
    // thread (h, r): channel nb + r, bytes [32 * blockIdx.y + 16h, +16) = the
    // words of warps 4h .. 4h + 3
    for (int tt = threadIdx.x; tt < 2 * COLS; tt += 256) {
        const int r = tt % COLS, h = tt / COLS;
        const int nn = nb + r;
        const int byte0 = blockIdx.y * 32 + 16 * h;  // a multiple of 16, as is ldw8
        if (nn < N && byte0 < ldw8)
            *reinterpret_cast<uint4 *>(Wq + (size_t)nn * ldw8 + byte0) =
                make_uint4(pk[4 * h][r], pk[4 * h + 1][r], pk[4 * h + 2][r], pk[4 * h + 3][r]);
    }
}

// Weight pass 3: turn the abs-max bits into the scale, in place.
template <int QMAX = 7>
__global__ void k_weight_scale_finalize(float *__restrict__ sw, int N) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n < N) {
        unsigned bits = reinterpret_cast<unsigned *>(sw)[n];
        sw[n] = weight_scale_from_amax<QMAX>(bits);
    }
}

// ---------------------------------------------------------------------------
// Activation quantization: one block per row (grid-stride over rows).
// The row is read once into registers (VPT floats per thread; longer rows
// are re-read for the quantization pass), its abs-max reduced with warp
// shuffles and then across warps, and the codes are stored 4 (or 8) at a time.
// Bytes K..ldq-1 of each row are written 0.
//
// PERM = false: natural k order (the public layout of a8_quantize_rows).
// PERM = true: inside every group of 8 consecutive k the bytes are stored as
// k0 k2 k4 k6 k1 k3 k5 k7 - the order in which the tensor-core kernel's
// weight unpack produces codes - so that kernel needs no byte permutes. Only
// used for the INT8 activations w4a8_linear keeps in its workspace.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float row_load(const float *__restrict__ x, int k, int K) {
    return k < K ? ld_dep(x + k) : 0.0f;
}

template <int U>
__device__ __forceinline__ void load_unit(const float *__restrict__ x, int k, int K, bool vec4, float (&v)[U]) {
#pragma unroll
    for (int h = 0; h < U / 4; ++h) {
        const int kk = k + 4 * h;
        if (vec4 && kk + 3 < K) {
            const float4 f = ld_dep_f4(x + kk);
            v[4 * h] = f.x; v[4 * h + 1] = f.y; v[4 * h + 2] = f.z; v[4 * h + 3] = f.w;
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) v[4 * h + b] = row_load(x, kk + b, K);
        }
    }
}

// Quantize one unit of U consecutive k (k0 = first k) and store it.
// `sum` accumulates the unit's codes (for the zero-point form's row sums).
template <int U, bool PERM>
__device__ __forceinline__ void store_unit(int8_t *__restrict__ row, int k0, int K, float s, const float (&v)[U],
                                           int &sum) {
    if constexpr (!PERM) {
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) w |= act_code8(v[b], s, k0 + b < K) << (8 * b);
        *reinterpret_cast<uint32_t *>(row + k0) = w;
        sum = __dp4a((int)w, 0x01010101, sum);
    } else {
        uint32_t even = 0, odd = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            even |= act_code8(v[2 * b], s, k0 + 2 * b < K) << (8 * b);
            odd |= act_code8(v[2 * b + 1], s, k0 + 2 * b + 1 < K) << (8 * b);
        }
        *reinterpret_cast<uint2 *>(row + k0) = make_uint2(even, odd);
        sum = __dp4a((int)even, 0x01010101, __dp4a((int)odd, 0x01010101, sum));
    }
}

template <int THREADS, int VPT, bool PERM>
__global__ void __launch_bounds__(THREADS)
k_act_quant(const float *__restrict__ X, int M, int K, int ldx,
            int8_t *__restrict__ Xq, int ldq, float *__restrict__ sx, int vec4, int32_t *__restrict__ rowsum) {
    constexpr int U = PERM ? 8 : 4;  // consecutive k per unit of work
    constexpr int G = VPT / U;       // units a thread keeps in registers
    static_assert(THREADS % 32 == 0 && THREADS <= 1024 && VPT % U == 0, "block shape");
    __shared__ float red[THREADS / 32];
    // X may be written by the previous kernel: wait for it. Only then let the
    // next kernel launch, so everything enqueued before this kernel has
    // completed when a dependent starts; the decode kernel relies on that to
    // stream its weights before its own griddepcontrol.wait (which returns
    // when this grid has finished). Every block triggers, so all of this grid
    // is resident before a dependent block can take an SM slot.
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool in_regs = K <= THREADS * VPT;
    const int units = ldq / U;  // ldq is a multiple of 16
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const float *x = X + (size_t)m * ldx;
        // unit u covers k = U*u .. U*u + U-1; thread t holds units t + i*THREADS
        float v[G][U];
        float amax = 0.0f;
        if (in_regs) {
#pragma unroll
            for (int i = 0; i < G; ++i) {
                load_unit<U>(x, U * (threadIdx.x + i * THREADS), K, vec4 != 0, v[i]);
#pragma unroll
                for (int b = 0; b < U; ++b) amax = fmaxf(amax, fabsf(v[i][b]));
            }
        } else {
            for (int k = threadIdx.x; k < K; k += THREADS) amax = fmaxf(amax, fabsf(ld_dep(x + k)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        float a = red[0];
#pragma unroll
        for (int i = 1; i < THREADS / 32; ++i) a = fmaxf(a, red[i]);
        const float s = act_scale_from_amax(a);
        if (threadIdx.x == 0) sx[m] = s;
        int8_t *row = Xq + (size_t)m * ldq;
        int sum = 0;
        if (in_regs) {
#pragma unroll
            for (int i = 0; i < G; ++i) {
                const int u = threadIdx.x + i * THREADS;
                if (u < units) store_unit<U, PERM>(row, U * u, K, s, v[i], sum);
            }
            for (int u = threadIdx.x + G * THREADS; u < units; u += THREADS) {
                float z[U];
#pragma unroll
                for (int b = 0; b < U; ++b) z[b] = 0.0f;
                store_unit<U, PERM>(row, U * u, K, s, z, sum);
            }
        } else {
            for (int u = threadIdx.x; u < units; u += THREADS) {
                float w[U];
                load_unit<U>(x, U * u, K, vec4 != 0, w);
                store_unit<U, PERM>(row, U * u, K, s, w, sum);
            }
        }
        __syncthreads();  // red is reused below and by the next row
        if (rowsum != nullptr) {
            // sum_k xq[m][k] for the zero-point form (pad codes are 0)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) red[warp] = __int_as_float(sum);
            __syncthreads();
            if (threadIdx.x == 0) {
                int t = 0;
#pragma unroll
                for (int i = 0; i < THREADS / 32; ++i) t += __float_as_int(red[i]);
                rowsum[m] = t;
            }
            __syncthreads();
        }
    }
}

}  // namespace w4a8
