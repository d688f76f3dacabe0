// Cluster K-split decode kernel: the whole few-row layer (steps 3-6 of "How it
// works" in the Keras guide "INT4 quantization in Keras": dynamic INT8
// quantization of the activation rows, INT4 -> INT8 unpack, INT8 x INT8 ->
// INT32, dequantization, bias, ReLU) in one launch, for at most 16 rows.
//
// With few activation rows the layer is a stream of the packed weights, and
// a short layer (a few MB) is bound by the chain of dependent launches rather
// than by bytes: what counts is how little work is left after the kernel's
// programmatic dependency wait. So the work is cut along K as well as N:
//  * a CTA owns 128 output channels (8 warps x 16) and one K slice of
//    ch x 128 k; the C CTAs that share a channel block form a thread-block
//    cluster (C <= 8) and cover K between them;
//  * each thread holds its weight bytes in registers, loaded before the
//    dependency wait when they are known to be final;
//  * after the wait a CTA reads only its K slice of the activation rows. With
//    float32 input it reduces the slice's row abs-max, the cluster's CTAs
//    exchange those partial maxima through distributed shared memory, and
//    every CTA derives the exact row scale sx = 127 / max|X[m,:]| and
//    quantizes its slice with the arithmetic of the activation pass (same
//    codes, same scales); the row maxima may also come from the producing
//    layer (per-16-channel parts of its output, see y_amax below);
//  * the slice's INT8 codes go to shared memory in the k-permuted order
//    k0 k2 k4 k6 k1 k3 k5 k7 of every 8 k, which is the order the 16 q nibble
//    masks produce, and the warps multiply on the integer MMA path
//    (mma.sync m16n8k32 s8, weights as A, tokens as B);
//  * the INT32 partial sums of the C slices meet in the CTA that owns the
//    channel group (warp w's group is owned by cluster rank w % C), which
//    shifts out the 16 of the nibble trick, dequantizes and stores.
// Every barrier is a hardware (CTA or cluster) barrier that all threads reach
// on every path, so nothing waits on memory written by another grid.
//
// Optionally (layer chaining) the epilogue also writes, for every output row
// m and every 16 consecutive output channels p, the abs-max of the stored
// float32 outputs, y_amax[m][p]: the next layer's row abs-max is the max over
// p, so it can quantize its input without a reduction over the row.
#pragma once

#include "common.cuh"
#include "decode_bulk.cuh"
#include "linear_simt.cuh"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace dsplit {

constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;
constexpr int CTA_CHANNELS = 16 * WARPS;  // output channels per CTA
constexpr int MAX_CLUSTER = 8;            // portable cluster size
constexpr int MAX_CH = 8;                 // 128-k chunks per CTA (register budget of the weights)
constexpr int MAX_TOK = 16;

// Where the activation rows come from.
//  IN_Q        : INT8 rows Xq [M][ldq] and scales sx [M] (natural k order);
//  IN_F32      : float32 rows X [M][ldx]; the cluster reduces the row abs-max;
//  IN_F32_PARTS: float32 rows X plus x_amax [M][x_parts], per-part abs-maxes
//                whose max over the parts is the row abs-max.
enum { IN_Q = 0, IN_F32 = 1, IN_F32_PARTS = 2 };

struct Params {
    const int8_t *Xq;
    const float *sx;
    int ldq;
    const float *X;
    int ldx;
    int vec4;  // X rows 16-byte aligned with ldx % 4 == 0
    const float *x_amax;
    int x_parts;
    int M, K;
    const uint8_t *Wp;
    int ldp;
    const float *sw;
    int N;
    const float *bias;
    unsigned flags;
    void *Y;
    int ldy;
    float *y_amax;  // [M][y_parts] or null
    int y_parts;
    int ch;  // 128-k chunks per CTA
    ZpArgs zpa;  // zero-point correction (null zp: none)
};

// Shared-memory row pitch of the INT8 slice: ch x 128 bytes + 16, so the
// 16-byte reads of a quarter-warp (two rows, four 32-byte offsets) hit 32
// distinct banks.
__host__ __device__ inline int xs_pitch(int ch) { return 128 * ch + 16; }
// Receive buffer of the cluster reduction: per owned warp slot, per source
// rank, per lane, 4 x NTG partial sums.
__host__ __device__ inline int recv_ints(int C, int tok) { return ((WARPS + C - 1) / C) * C * 32 * (tok / 2); }

// Eight floats X[r][k..k+7] (zeros past K).
__device__ __forceinline__ void load8(const float *row, int k, int K, int vec4, float (&v)[8]) {
#pragma unroll
    for (int b = 0; b < 8; ++b) v[b] = 0.0f;
    if (k >= K) return;
    if (vec4 && k + 7 < K) {
        const float4 f0 = ld_dep_f4(row + k), f1 = ld_dep_f4(row + k + 4);
        v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
        v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
    } else {
#pragma unroll
        for (int b = 0; b < 8; ++b)
            if (k + b < K) v[b] = ld_dep(row + k + b);
    }
}

// NTG: token groups of 8 (M <= 8 NTG). IN: activation source. EARLY: the
// weights, their scales and the bias are final at launch (behind this
// library's activation pass, or W4A8_STATIC_WEIGHTS), so they are read before
// the dependency wait. CHMAX: register capacity in 128-k chunks (ch <= CHMAX).
template <int NTG, int IN, bool EARLY, int CHMAX>
__global__ void __launch_bounds__(THREADS)
k_decode_split(const __grid_constant__ Params p) {
    constexpr int TOK = 8 * NTG;
    __shared__ unsigned s_amax[TOK];               // this slice's row abs-max (float bits)
    __shared__ float s_part[MAX_CLUSTER][TOK];     // every slice's row abs-max, written by its CTA
    __shared__ float s_sx[TOK];
    extern __shared__ __align__(16) uint8_t dsm[];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
    const uint32_t C = ptx::cluster_nctarank();
    const uint32_t rank = ptx::cluster_ctarank();
    const bool clustered = C > 1;
    const int ch = p.ch;
    const int pitch = xs_pitch(ch);
    int8_t *xs = reinterpret_cast<int8_t *>(dsm);                        // [TOK][pitch], permuted k
    int32_t *recv = reinterpret_cast<int32_t *>(dsm + TOK * pitch);     // see recv_ints
    const int k0 = (int)rank * 128 * ch;                                 // first k of this CTA's slice
    const int n0 = ((int)blockIdx.y * WARPS + warp) * 16;                // this warp's channel group
    const int M = p.M, K = p.K, N = p.N;

    // Phase 0 of the cluster barrier: "this CTA is running". Its wait comes
    // before the first access to a peer's shared memory.
    if (clustered) ptx::cluster_arrive_relaxed();
    griddep_launch_dependents();

    // Weights: thread (g, t) holds bytes [64 c + 16 t, +16) of the slice of
    // rows n0 + g and n0 + g + 8 for its chunks c < ch (bytes past the packed
    // row's kp and rows past N read as zeros).
    const int kp = packed_row_bytes(K);
    const int nA = n0 + g, nB = n0 + g + 8;
    const bool okA = nA < N, okB = nB < N;
    const uint8_t *wA = p.Wp + (size_t)(okA ? nA : 0) * p.ldp + k0 / 2 + 16 * t;
    const uint8_t *wB = p.Wp + (size_t)(okB ? nB : 0) * p.ldp + k0 / 2 + 16 * t;
    uint4 wa[CHMAX], wb[CHMAX];
    const bool has_bias = p.bias != nullptr && (p.flags & W4A8_OUT_MASK) != W4A8_OUT_S32;
    float swA = 1.0f, swB = 1.0f, bA = 0.0f, bB = 0.0f;
    auto load_weights = [&]() {
#pragma unroll
        for (int c = 0; c < CHMAX; ++c) {
            const bool in = c < ch && k0 / 2 + 64 * c + 16 * t < kp;
            const uint4 z = make_uint4(0, 0, 0, 0);
            wa[c] = (in && okA) ? ld_stream_v4(wA + 64 * c) : z;
            wb[c] = (in && okB) ? ld_stream_v4(wB + 64 * c) : z;
        }
        if (okA) swA = ld_dep(p.sw + nA);
        if (okB) swB = ld_dep(p.sw + nB);
        if (has_bias) {
            if (okA) bA = ld_dep(p.bias + nA);
            if (okB) bB = ld_dep(p.bias + nB);
        }
    };
    if constexpr (EARLY) {
        load_weights();
    } else if (lane < 16 && n0 + lane < N) {
        // bring this warp's rows of the slice into L2 without reading them
        const int bytes = min(64 * ch, kp - k0 / 2);
        if (bytes > 0) prefetch_l2_bulk(p.Wp + (size_t)(n0 + lane) * p.ldp + k0 / 2, (uint32_t)bytes);
    }
    griddep_wait();
    if constexpr (!EARLY) load_weights();

    // ------------------------------------------------ activation slice
    bool waited0 = false;
    if constexpr (IN == IN_Q) {
        // 16-byte pieces of the slice, byte-permuted into xs (k >= ldq or
        // rows >= M read as zeros); loads batched ahead of the stores
        const int per = 8 * ch;
        constexpr int QB = 4;
        for (int base = tid; base < TOK * per; base += THREADS * QB) {
            uint4 v[QB];
#pragma unroll
            for (int j = 0; j < QB; ++j) {
                const int u = base + j * THREADS;
                const int r = u / per, kk = k0 + 16 * (u - r * per);
                v[j] = make_uint4(0, 0, 0, 0);
                if (u < TOK * per && r < M && kk < p.ldq) {
                    const uint4 x = ld_dep_v4(p.Xq + (size_t)r * p.ldq + kk);
                    v[j] = make_uint4(__byte_perm(x.x, x.y, 0x6420), __byte_perm(x.x, x.y, 0x7531),
                                      __byte_perm(x.z, x.w, 0x6420), __byte_perm(x.z, x.w, 0x7531));
                }
            }
#pragma unroll
            for (int j = 0; j < QB; ++j) {
                const int u = base + j * THREADS;
                if (u < TOK * per) {
                    const int r = u / per;
                    *reinterpret_cast<uint4 *>(xs + r * pitch + 16 * (u - r * per)) = v[j];
                }
            }
        }
    } else {
        const int upr = 16 * ch;  // units of 8 floats per row of the slice
        constexpr int FB = 2;     // units per thread in flight
        if constexpr (IN == IN_F32) {
            // pass 1: this slice's abs-max of every row
            if (tid < TOK) s_amax[tid] = 0u;
            __syncthreads();
            const bool warp_rows = (upr % 32) == 0;  // a warp's 32 units then share one row
            for (int base = tid; base < M * upr; base += THREADS * FB) {
                float v[FB][8];
#pragma unroll
                for (int j = 0; j < FB; ++j) {
                    const int u = base + j * THREADS;
                    const int r = u / upr;
#pragma unroll
                    for (int b = 0; b < 8; ++b) v[j][b] = 0.0f;
                    if (u < M * upr) load8(p.X + (size_t)r * p.ldx, k0 + 8 * (u - r * upr), K, p.vec4, v[j]);
                }
#pragma unroll
                for (int j = 0; j < FB; ++j) {
                    const int u = base + j * THREADS;
                    float a = 0.0f;
#pragma unroll
                    for (int b = 0; b < 8; ++b) a = fmaxf(a, fabsf(v[j][b]));
                    if (warp_rows) {
                        const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
                        if (lane == 0 && u < M * upr) atomicMax(&s_amax[u / upr], m);
                    } else if (u < M * upr) {
                        atomicMax(&s_amax[u / upr], __float_as_uint(a));
                    }
                }
            }
            __syncthreads();
            // every CTA of the cluster learns every slice's maximum
            if (clustered) {
                ptx::cluster_wait_acquire();
                waited0 = true;
            }
            if (tid < TOK) {
                const float a = __uint_as_float(s_amax[tid]);
                if (clustered) {
                    const uint32_t la = ptx::smem_addr(&s_part[rank][tid]);
                    for (uint32_t r2 = 0; r2 < C; ++r2) ptx::st_cluster_f32(ptx::mapa_shared(la, r2), a);
                } else {
                    s_part[0][tid] = a;
                }
            }
            if (clustered) {
                ptx::cluster_arrive_release();
                ptx::cluster_wait_acquire();
            } else {
                __syncthreads();
            }
            if (tid < TOK) {
                float a = s_part[0][tid];
                for (uint32_t r2 = 1; r2 < C; ++r2) a = fmaxf(a, s_part[r2][tid]);
                s_sx[tid] = act_scale_from_amax(a);
            }
        } else {
            // the row abs-max is the max of the producer's parts
            for (int r = warp; r < TOK; r += WARPS) {
                float a = 0.0f;
                if (r < M) {
                    const float *pr = p.x_amax + (size_t)r * p.x_parts;
                    for (int j0 = 0; j0 < p.x_parts; j0 += 32 * 8) {
                        float v[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int j = j0 + 32 * u + lane;
                            v[u] = j < p.x_parts ? ld_dep(pr + j) : 0.0f;
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) a = fmaxf(a, v[u]);
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
                if (lane == 0) s_sx[r] = act_scale_from_amax(a);
            }
        }
        __syncthreads();
        // pass 2: quantize the slice (rows >= M and k >= K give code 0)
        for (int base = tid; base < TOK * upr; base += THREADS * FB) {
            float v[FB][8];
#pragma unroll
            for (int j = 0; j < FB; ++j) {
                const int u = base + j * THREADS;
                const int r = u / upr;
#pragma unroll
                for (int b = 0; b < 8; ++b) v[j][b] = 0.0f;
                if (u < TOK * upr && r < M) load8(p.X + (size_t)r * p.ldx, k0 + 8 * (u - r * upr), K, p.vec4, v[j]);
            }
#pragma unroll
            for (int j = 0; j < FB; ++j) {
                const int u = base + j * THREADS;
                if (u < TOK * upr) {
                    const int r = u / upr, c8 = u - r * upr;
                    const uint2 q = r < M ? dbulk::act_codes8_perm(v[j], s_sx[r], k0 + 8 * c8, K) : make_uint2(0, 0);
                    *reinterpret_cast<uint2 *>(xs + r * pitch + 8 * c8) = q;
                }
            }
        }
    }
    __syncthreads();

    // ------------------------------------------------ product
    // MMA q of chunk c takes word q of the thread's 16 weight bytes, i.e.
    // k = 128 c + 32 t + 8 q .. +7 of the slice: 16 q of the even k (low
    // nibbles) to A slots 4t.., of the odd k to 16 + 4t..; the INT8 slice
    // holds the same k as the even/odd words of one permuted 8-k group.
    int32_t acc[NTG][4][4];
#pragma unroll
    for (int i = 0; i < NTG; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q][0] = acc[i][q][1] = acc[i][q][2] = acc[i][q][3] = 0;
#pragma unroll
    for (int c = 0; c < CHMAX; ++c) {
        if (c >= ch) break;
        const uint32_t pa[4] = {wa[c].x, wa[c].y, wa[c].z, wa[c].w};
        const uint32_t pb[4] = {wb[c].x, wb[c].y, wb[c].z, wb[c].w};
#pragma unroll
        for (int i = 0; i < NTG; ++i) {
            const int8_t *xp = xs + (8 * i + g) * pitch + 128 * c + 32 * t;
            const uint4 x0 = ptx::lds128(xp), x1 = ptx::lds128(xp + 16);
            const uint32_t xe[4] = {x0.x, x0.z, x1.x, x1.z}, xo[4] = {x0.y, x0.w, x1.y, x1.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t alo = (pa[q] << 4) & 0xF0F0F0F0u, ahi = pa[q] & 0xF0F0F0F0u;
                const uint32_t blo = (pb[q] << 4) & 0xF0F0F0F0u, bhi = pb[q] & 0xF0F0F0F0u;
                mma_s8_16832(acc[i][q], alo, blo, ahi, bhi, xe[q], xo[q]);
            }
        }
    }
    int32_t tot[NTG][4];
#pragma unroll
    for (int i = 0; i < NTG; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) tot[i][j] = acc[i][0][j] + acc[i][1][j] + acc[i][2][j] + acc[i][3][j];

    // ------------------------------------------------ cluster reduction
    if (clustered) {
        if (!waited0) ptx::cluster_wait_acquire();
        const uint32_t owner = (uint32_t)warp % C, slot = (uint32_t)warp / C;
        const uint32_t la = ptx::smem_addr(recv + ((slot * C + rank) * 32 + lane) * (4 * NTG));
        const uint32_t ra = ptx::mapa_shared(la, owner);
#pragma unroll
        for (int i = 0; i < NTG; ++i) ptx::st_cluster_v4(ra + 16 * i, tot[i][0], tot[i][1], tot[i][2], tot[i][3]);
        ptx::cluster_arrive_release();
        ptx::cluster_wait_acquire();
        if (owner != rank) return;  // no remote access follows: safe to leave
#pragma unroll
        for (int i = 0; i < NTG; ++i) tot[i][0] = tot[i][1] = tot[i][2] = tot[i][3] = 0;
        for (uint32_t r2 = 0; r2 < C; ++r2) {
            const int32_t *src = recv + ((slot * C + r2) * 32 + lane) * (4 * NTG);
#pragma unroll
            for (int i = 0; i < NTG; ++i) {
                const uint4 v = ptx::lds128(src + 4 * i);
                tot[i][0] += (int32_t)v.x;
                tot[i][1] += (int32_t)v.y;
                tot[i][2] += (int32_t)v.z;
                tot[i][3] += (int32_t)v.w;
            }
        }
    }

    // ------------------------------------------------ epilogue
    // tot[i][e] : channel nA, token 8 i + 2 t + e;  tot[i][2 + e]: channel nB.
    const unsigned fmt = p.flags & W4A8_OUT_MASK;
    const bool relu = (p.flags & W4A8_RELU) != 0;
    const bool emit = p.y_amax != nullptr;
#pragma unroll
    for (int i = 0; i < NTG; ++i) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int m = 8 * i + 2 * t + e;
            const bool m_ok = m < M;
            float sxm = 1.0f;
            if (m_ok) sxm = IN == IN_Q ? ld_dep(p.sx + m) : s_sx[m];
            float amx = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = h ? nB : nA;
                const bool ok = m_ok && (h ? okB : okA);
                if (!ok) continue;
                const int32_t a = zp_fix(tot[i][2 * h + e] >> 4, p.zpa, m, n);  // >> 4 exact: terms are multiples of 16
                const size_t off = (size_t)m * (size_t)p.ldy + (size_t)n;
                if (fmt == W4A8_OUT_S32) {
                    static_cast<int32_t *>(p.Y)[off] = a;
                } else {
                    const float y = dequant_value(a, sxm, h ? swB : swA, has_bias, h ? bB : bA, relu);
                    if (fmt == W4A8_OUT_BF16)
                        static_cast<__nv_bfloat16 *>(p.Y)[off] = __float2bfloat16_rn(y);
                    else
                        static_cast<float *>(p.Y)[off] = y;
                    amx = fmaxf(amx, fabsf(y));
                }
            }
            if (emit) {
                // the 16 channels of this group for token m sit on the 8 lanes with this t
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, 4));
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, 8));
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, 16));
                if (g == 0 && m_ok && n0 < N) p.y_amax[(size_t)m * p.y_parts + n0 / 16] = amx;
            }
        }
    }
}

// ------------------------------------------------------------- host side ---

struct Plan {
    bool ok = false;
    int C = 1, ch = 1, chmax = 2, nblk = 0, tok = 8;
    size_t smem = 0;
};

// K slices: the packed row's 64-byte chunks (128 k each) split over at most
// MAX_CLUSTER CTAs of at most MAX_CH chunks; the slice count drops any rank
// that would get no chunk.
inline Plan plan(int M, int K, int N) {
    Plan s;
    if (M < 1 || M > MAX_TOK || K < 1 || N < 1) return s;
    const int nchunks = (packed_row_bytes(K) + 63) / 64;
    if (nchunks > MAX_CLUSTER * MAX_CH) return s;
    int C = nchunks < MAX_CLUSTER ? nchunks : MAX_CLUSTER;
    const int ch = (nchunks + C - 1) / C;
    C = (nchunks + ch - 1) / ch;
    const long long nblk = ((long long)N + CTA_CHANNELS - 1) / CTA_CHANNELS;
    if (nblk > 65535) return s;
    s.C = C;
    s.ch = ch;
    s.chmax = ch <= 2 ? 2 : (ch <= 4 ? 4 : 8);
    s.nblk = (int)nblk;
    s.tok = M <= 8 ? 8 : 16;
    s.smem = (size_t)s.tok * xs_pitch(ch) + (size_t)recv_ints(C, s.tok) * sizeof(int32_t);
    s.ok = true;
    return s;
}

template <int NTG, int IN, bool EARLY, int CHMAX>
inline cudaError_t launch_t(const Plan &pl, const Params &p, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.C, pl.nblk);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (pl.C > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)pl.C;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, k_decode_split<NTG, IN, EARLY, CHMAX>, p);
}

template <int NTG, int IN, bool EARLY>
inline cudaError_t launch_ch(const Plan &pl, const Params &p, cudaStream_t s) {
    if (pl.chmax == 2) return launch_t<NTG, IN, EARLY, 2>(pl, p, s);
    if (pl.chmax == 4) return launch_t<NTG, IN, EARLY, 4>(pl, p, s);
    return launch_t<NTG, IN, EARLY, 8>(pl, p, s);
}

template <int IN>
inline cudaError_t launch(const Plan &pl, const Params &p, bool early, cudaStream_t s) {
    if (pl.tok == 8) return early ? launch_ch<1, IN, true>(pl, p, s) : launch_ch<1, IN, false>(pl, p, s);
    return early ? launch_ch<2, IN, true>(pl, p, s) : launch_ch<2, IN, false>(pl, p, s);
}

}  // namespace dsplit
}  // namespace w4a8
