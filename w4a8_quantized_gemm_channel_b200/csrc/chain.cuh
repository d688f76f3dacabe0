// Layer chaining: a Dense layer whose float32 input comes from the previous
// layer (the Keras guide "INT4 quantization in Keras", "Quantize a minimal
// functional model": Dense -> ReLU -> Dense, each layer quantizing its own
// input dynamically, step 3 of "How it works"). The activation step needs each
// input row's abs-max; the producing layer can emit it as per-16-channel
// parts y_amax[m][p] = max |Y[m][16 p .. 16 p + 15]|, whose max over p is the
// row abs-max exactly.
//
//  * k_linear_generic_f32: the generic product with the activation step
//    inside (tiny layers): the block derives the row scale from the parts, or
//    reduces the row itself, and every thread quantizes X on the fly with the
//    activation pass's arithmetic; optionally emits its own output's parts.
//  * k_row_amax_parts: the parts of a finished float32 output, for the paths
//    whose product kernels do not emit them.
#pragma once

#include "common.cuh"

namespace w4a8 {
namespace chain {

constexpr int GEN_THREADS = 128;

// grid = (ceil(N / 128), min(M, 65535)); one thread per output channel, rows
// blockIdx.y, + gridDim.y, ...
__global__ void __launch_bounds__(GEN_THREADS)
k_linear_generic_f32(const float *X, int M, int K, int ldx, const float *x_amax, int x_parts,
                     const uint8_t *Wp, int ldp, const float *sw, int N, const float *bias, unsigned flags,
                     float *Y, int ldy, float *y_amax, int y_parts) {
    __shared__ float s_red[GEN_THREADS / 32];
    griddep_launch_dependents();
    griddep_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = blockIdx.x * GEN_THREADS + tid;
    const bool n_ok = n < N;
    const float swn = n_ok ? ld_dep(sw + n) : 1.0f;
    const float bn = (bias != nullptr && n_ok) ? ld_dep(bias + n) : 0.0f;
    const uint8_t *wr = Wp + (size_t)(n_ok ? n : 0) * ldp;
    const bool relu = (flags & W4A8_RELU) != 0;
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
        const float *xr = X + (size_t)m * ldx;
        // the row scale (step 3): abs-max of the row, from the parts or the row
        float a = 0.0f;
        if (x_amax != nullptr) {
            for (int j = tid; j < x_parts; j += GEN_THREADS) a = fmaxf(a, ld_dep(x_amax + (size_t)m * x_parts + j));
        } else {
            for (int k = tid; k < K; k += GEN_THREADS) a = fmaxf(a, fabsf(ld_dep(xr + k)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (lane == 0) s_red[warp] = a;
        __syncthreads();
        a = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
        __syncthreads();  // s_red is rewritten for the next row
        const float s = act_scale_from_amax(a);
        // steps 4-5: codes of X times the channel's nibbles (byte k/2: code k
        // in the low nibble, k + 1 in the high one)
        int32_t acc = 0;
        if (n_ok) {
            for (int k = 0; k < K; k += 2) {
                const uint32_t b = ld_dep_u8(wr + (k >> 1));
                acc += (int)(int8_t)act_code8(ld_dep(xr + k), s, true) * ((int)((b & 0xFu) ^ 8u) - 8);
                if (k + 1 < K) acc += (int)(int8_t)act_code8(ld_dep(xr + k + 1), s, true) * ((int)((b >> 4) ^ 8u) - 8);
            }
        }
        // step 6 and the Dense epilogue
        const float y = n_ok ? dequant_value(acc, s, swn, bias != nullptr, bn, relu) : 0.0f;
        if (n_ok) Y[(size_t)m * ldy + n] = y;
        if (y_amax != nullptr) {
            float am = fabsf(y);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
            if ((tid & 15) == 0 && n_ok) y_amax[(size_t)m * y_parts + n / 16] = am;
        }
    }
}

// grid = (ceil(y_parts / 128), min(M, 65535)); one thread per part.
__global__ void __launch_bounds__(128)
k_row_amax_parts(const float *Y, int M, int N, int ldy, float *y_amax, int y_parts) {
    griddep_launch_dependents();
    griddep_wait();
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= y_parts) return;
    const int cnt = min(16, N - 16 * p);
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
        const float *yr = Y + (size_t)m * ldy + 16 * p;
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = j < cnt ? ld_dep(yr + j) : 0.0f;
        float a = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(v[j]));
        y_amax[(size_t)m * y_parts + p] = a;
    }
}

}  // namespace chain
}  // namespace w4a8
