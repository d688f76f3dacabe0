// Single-pass weight quantize+pack (Keras guide "INT4 quantization in Keras",
// "How it works", steps 1-2): per output channel n, sw[n] = 7 / max_k |W[k][n]|
// (1 for an all-zero column) and q = clamp(rne(W[k][n] * sw[n]), -8, 7),
// packed two codes per byte along K, even k in the low nibble. QB = 8 is the
// W8A8 form the guide's closing paragraph names: sw = 127 / abs-max,
// q in [-127, 127], one byte per code.
//
// The two-pass form (k_col_absmax, then k_quant_pack) reads W twice from
// DRAM. Here a cluster of C <= 8 CTAs owns a panel of 32 output channels
// (128 bytes of every W row): CTA r loads rows [r Ks, (r+1) Ks) of the panel
// into shared memory with TMA (boxes of 256 rows x 128 bytes; rows past K
// and columns past N read as zero), takes the per-column abs-max of its
// slice, and the cluster combines the C partial maxima through distributed
// shared memory. Every CTA then quantizes and packs its slice straight from
// shared memory, so W is read from DRAM once. The arithmetic is the two-pass
// form's (same scale function, same rounding), so the outputs are identical.
//
// Layouts this serves: W 16-byte aligned with ldw a multiple of 4 (the TMA
// tensor map needs 16-byte row strides) and slices of at most 1536 rows
// (K <= 12288); the host takes the two-pass form otherwise.
#pragma once

#include "gemm_tc.cuh"
#include "quant_kernels.cuh"

namespace w4a8 {
namespace qpp {

constexpr int COLS = 32;            // output channels per panel: 128 bytes of a W row
constexpr int BOX_ROWS = 256;       // rows per TMA box
constexpr int MAX_CLUSTER = 8;
constexpr int MAX_SLICE = 1536;     // rows per CTA: 192 KB of shared memory
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;

struct Plan {
    int C;    // CTAs per panel (the cluster)
    int Ks;   // rows per CTA, a multiple of BOX_ROWS
    bool ok;
};

// About 512 rows per CTA (64 KB, three CTAs per SM) up to eight CTAs per
// panel; longer slices beyond that, up to MAX_SLICE.
inline Plan plan(int K) {
    int C = (K + 511) / 512;
    C = C < 1 ? 1 : (C > MAX_CLUSTER ? MAX_CLUSTER : C);
    const int Ks = ((K + C - 1) / C + BOX_ROWS - 1) / BOX_ROWS * BOX_ROWS;
    return {C, Ks, K >= 1 && Ks <= MAX_SLICE};
}

inline size_t smem_bytes(int Ks) {
    // tile [Ks][COLS], pmax [COLS], red [WARPS][COLS], scale [COLS], barrier,
    // abort flag, and the alignment slack of the 1024-aligned base
    return (size_t)Ks * COLS * 4 + (2 + WARPS) * COLS * 4 + 16 + 1024;
}

// QB: bits per code (4 or 8). grid = (ceil(N / COLS), C), cluster (1, C, 1),
// block = THREADS.
template <int QB>
__global__ void __launch_bounds__(THREADS)
k_quant_pack_panel(const __grid_constant__ CUtensorMap tm_w, int K, int N, int Ks, uint8_t *__restrict__ Wp, int ldp,
                   float *__restrict__ sw) {
    static_assert(QB == 4 || QB == 8, "INT4 or INT8 codes");
    constexpr int QMAX = QB == 4 ? 7 : 127;
    constexpr int QMIN = QB == 4 ? -8 : -127;
    constexpr int PER_WORD = 32 / QB;           // codes per 32-bit word
    constexpr int WORDS = 64 / PER_WORD;        // words per 64 rows
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float(*tile)[COLS] = reinterpret_cast<float(*)[COLS]>(base);
    float *pmax = reinterpret_cast<float *>(base + (size_t)Ks * COLS * 4);
    float(*red)[COLS] = reinterpret_cast<float(*)[COLS]>(pmax + COLS);
    float *scale = reinterpret_cast<float *>(red + WARPS);
    uint64_t *bar = reinterpret_cast<uint64_t *>(scale + COLS);
    int *abort_flag = reinterpret_cast<int *>(bar + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = (int)gridDim.y;
    const int r = (int)blockIdx.y;  // the cluster spans gridDim.y, so this is the CTA's rank in it
    const int n0 = (int)blockIdx.x * COLS;
    const int k0 = r * Ks;

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_w);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)Ks * COLS * 4);
        for (int b = 0; b < Ks / BOX_ROWS; ++b)
            ptx::tma_load_2d(&tile[b * BOX_ROWS][0], &tm_w, n0, k0 + b * BOX_ROWS, bar);
    }
    const bool ok = ptx::mbar_wait(bar, 0, abort_flag);

    // per-column abs-max of this slice (rows past K are zero)
    float m = 0.0f;
    if (ok)
        for (int i = warp; i < Ks; i += WARPS) m = fmaxf(m, fabsf(tile[i][lane]));
    red[warp][lane] = m;
    __syncthreads();
    if (warp == 0) {
        float a = red[0][lane];
#pragma unroll
        for (int w = 1; w < WARPS; ++w) a = fmaxf(a, red[w][lane]);
        pmax[lane] = a;
    }
    // every CTA's partial maxima are written before any CTA reads them
    ptx::cluster_arrive_release();
    ptx::cluster_wait_acquire();
    if (warp == 0) {
        float a = 0.0f;
        for (int q = 0; q < C; ++q) {
            float v;
            asm volatile("ld.shared::cluster.f32 %0, [%1];"
                         : "=f"(v)
                         : "r"(ptx::mapa_shared(ptx::smem_addr(pmax + lane), (uint32_t)q))
                         : "memory");
            a = fmaxf(a, v);
        }
        const float s = weight_scale_from_amax<QMAX>(__float_as_uint(a));
        scale[lane] = s;
        if (r == 0 && n0 + lane < N) sw[n0 + lane] = s;
    }
    __syncthreads();

    // quantize and pack: thread (warp, lane) takes channel n0 + lane and 64
    // consecutive rows per step: 64 codes = 32 (INT4) or 64 (INT8) bytes,
    // stored 16 bytes at a time
    const int n = n0 + lane;
    const float s = scale[lane];
    if (ok && n < N) {
        for (int j = warp; j < Ks / 64; j += WARPS) {
            uint32_t word[WORDS];
#pragma unroll
            for (int g = 0; g < WORDS; ++g) {
                uint32_t wv = 0;
#pragma unroll
                for (int i = 0; i < PER_WORD; ++i) {
                    const float v = tile[64 * j + PER_WORD * g + i][lane];
                    const int q = clampi(__float2int_rn(__fmul_rn(v, s)), QMIN, QMAX);
                    wv |= ((uint32_t)q & ((1u << QB) - 1u)) << (QB * i);
                }
                word[g] = wv;
            }
            const int byte0 = (k0 + 64 * j) * QB / 8;  // a multiple of 32; ldp is a multiple of 16
            uint8_t *dst = Wp + (size_t)n * ldp + byte0;
#pragma unroll
            for (int h = 0; h < WORDS / 4; ++h)
                if (byte0 + 16 * h < ldp)
                    *reinterpret_cast<uint4 *>(dst + 16 * h) =
                        make_uint4(word[4 * h], word[4 * h + 1], word[4 * h + 2], word[4 * h + 3]);
        }
    }
    // bytes of the packed rows beyond the cluster's rows (a row stride wider
    // than the codes need) are zero
    const int tail0 = C * Ks * QB / 8;
    if (r == C - 1 && tail0 < ldp) {
        const int chunks = (ldp - tail0) / 16;
        for (int t = threadIdx.x; t < COLS * chunks; t += THREADS) {
            const int c = t % COLS, h = t / COLS;
            if (n0 + c < N) *reinterpret_cast<uint4 *>(Wp + (size_t)(n0 + c) * ldp + tail0 + 16 * h) = make_uint4(0, 0, 0, 0);
        }
    }
    // a load this CTA gave up waiting for lands before the CTA exits
    if (!ok && threadIdx.x == 0) ptx::mbar_wait_drain(bar, 0);
    // no CTA leaves while another may still read its partial maxima
    ptx::cluster_arrive_release();
    ptx::cluster_wait_acquire();
}

// Whether the single-pass form serves this layout.
inline bool eligible(const float *W, int K, int ldw) {
    return plan(K).ok && (reinterpret_cast<uintptr_t>(W) & 15) == 0 && ldw % 4 == 0 && tc::encode_fn() != nullptr;
}

template <int QB>
inline w4a8_status launch(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp, float *sw,
                          cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(k_quant_pack_panel<QB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem_bytes(MAX_SLICE));
    });
    if (attr_err != cudaSuccess) return W4A8_ERR_CUDA;
    const Plan p = plan(K);
    if (!p.ok) return W4A8_ERR_UNSUPPORTED;
    CUtensorMap tm;
    if (!tc::make_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, W, (uint64_t)N, (uint64_t)K, (uint64_t)ldw * 4, COLS,
                         BOX_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return W4A8_ERR_CUDA;
    const long long panels = (N + COLS - 1) / COLS;
    if (panels > 0x7fffffffLL) return W4A8_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)panels, (unsigned)p.C);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem_bytes(p.Ks);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)p.C;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_quant_pack_panel<QB>, tm, K, N, p.Ks, Wp, ldp, sw);
    return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

}  // namespace qpp
}  // namespace w4a8
