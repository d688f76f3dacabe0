// extern "C" entry points of libw4a8.so: argument checks, workspace layout,
// kernel selection and launches. Declarations and contracts: include/w4a8.h.
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>

#include "w4a8.h"
#include "common.cuh"
#include "quant_kernels.cuh"
#include "linear_simt.cuh"
#include "linear_w8.cuh"
#include "zero_point.cuh"
#include "group_wise.cuh"
#include "decode_bulk.cuh"
#include "decode_split.cuh"
#include "chain.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc_grp.cuh"
#include "gemm_tc_pair.cuh"
#include "quant_pack_panel.cuh"

namespace w4a8 {
namespace {

thread_local unsigned t_last_path = 0;
thread_local unsigned t_last_launches = 0;
thread_local const char *t_last_kernel = "";

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

struct DeviceInfo {
    int sm_count = 0;
    int major = 0;
    bool ok = false;
};

// Per-device properties, read once per device.
const DeviceInfo &device_info() {
    static std::mutex mu;
    static DeviceInfo infos[64];
    static bool done[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        static DeviceInfo none;
        return none;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess)
            d.ok = (d.major == 10);
        infos[dev] = d;
        done[dev] = true;
    }
    return infos[dev];
}

// Launch with the programmatic-stream-serialization attribute, so a kernel
// may begin its prologue while its predecessor in the stream finishes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

w4a8_status from_cuda(cudaError_t e) { return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA; }

struct Workspace {
    int8_t *xq;
    float *sx;
    int ldq;
};

size_t workspace_bytes_for(int M, int K, int *ldq_out) {
    const int ldq = round_up(K, 16);
    if (ldq_out) *ldq_out = ldq;
    const size_t xq_bytes = ((size_t)M * (size_t)ldq + 255) / 256 * 256;
    return xq_bytes + (size_t)M * sizeof(float) + 256;
}

Workspace carve_workspace(void *ws, int M, int K) {
    Workspace w;
    workspace_bytes_for(M, K, &w.ldq);
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255);
    w.xq = reinterpret_cast<int8_t *>(base);
    base += ((size_t)M * (size_t)w.ldq + 255) / 256 * 256;
    w.sx = reinterpret_cast<float *>(base);
    return w;
}

w4a8_status check_common(int M, int K, int N, const uint8_t *Wp, int ldp, const float *sw,
                         const float *bias, unsigned flags, const void *Y, int ldy) {
    if (K < 1 || K > W4A8_MAX_K || N < 1 || M < 0) return W4A8_ERR_INVALID_ARG;
    if (!Wp || !sw || (!Y && M > 0)) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(Wp) || ldp < (K + 1) / 2 || ldp % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (ldy < N || !aligned4(sw) || (bias && !aligned4(bias))) return W4A8_ERR_INVALID_ARG;
    const unsigned fmt = flags & W4A8_OUT_MASK;
    if (fmt == (W4A8_OUT_BF16 | W4A8_OUT_S32)) return W4A8_ERR_INVALID_ARG;
    if (fmt == W4A8_OUT_S32 && (bias || (flags & W4A8_RELU))) return W4A8_ERR_INVALID_ARG;
    const size_t esz = fmt == W4A8_OUT_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(Y) & (esz - 1)) != 0) return W4A8_ERR_INVALID_ARG;
    if (flags & ~(W4A8_RELU | W4A8_OUT_MASK | W4A8_STATIC_WEIGHTS | W4A8_PATH_MASK)) return W4A8_ERR_INVALID_ARG;
    return W4A8_OK;
}

// The family (generic, decode, tensor core) of a path value: the forced
// decode kernels belong to the decode family.
inline unsigned path_family(unsigned path) {
    if (path == W4A8_PATH_TC_PAIR) return W4A8_PATH_TC;
    return path >= W4A8_PATH_DECODE_RING ? W4A8_PATH_DECODE : path;
}

// Kernel selection by shape. Few rows: the layer is a weight stream, so the
// decode kernel; many rows: the tensor-core GEMM; tiny problems: generic.
unsigned choose_path(int M, int K, int N, unsigned flags) {
    const unsigned forced = flags & W4A8_PATH_MASK;
    if (forced) return forced;
    const double work = (double)M * (double)N * (double)K;
    if (work < 65536.0) return W4A8_PATH_GENERIC;
    if (M <= 16) return W4A8_PATH_DECODE;
    if (tc_supported(M, K, N)) return W4A8_PATH_TC;
    return W4A8_PATH_DECODE;
}

// The tensor-core product on a CTA pair (k_gemm_tc_pair) rather than on one
// SM (k_gemm_tc): measured on B200 it is faster from M = 2048 rows up
// (1987 against 1893 TOPS at M = 2048, K = 4096, N = 11008; 2050 against
// 1805 at K = 11008, N = 4096; 2030 against 1970 at M = 8192) and slower at
// M = 512 (1147 against 1259), where its 160-token tiles leave the last round
// of the grid mostly idle.
bool pair_preferred(int M, int K, int N) {
    return M >= 1024 && N >= 512 && K <= tc::TC_X16_MAX_K;
}

// Kernels that take more than the default 48 KB of shared memory need the
// limit raised once per device.
bool raise_smem_limit(const void *kern, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, bool> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(kern, dev);
    if (done.count(key)) return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done[key] = true;
    return true;
}

// The persistent decode kernel (a TMA ring of weight stages) serves M <= 8
// when its ring and the activation rows fit the shared-memory budget, except
// where registers_beat_ring hands a short layer to k_linear_decode.
struct RingPlan {
    bool ok = false;
    int grid = 0, ring_n = 0;
    size_t smem = 0;
};

// Grid and ring for a layer. A block needs ring_n stages next to the INT8
// rows, within dbulk::SMEM_BUDGET. Short layers (at most two groups per SM):
// one group per block if two launches' blocks still fit an SM (so the next
// launch overlaps this one), else one block per SM. Long layers: two blocks
// per SM, each walking many groups.
RingPlan ring_plan(int M, int K, int N) {
    RingPlan p;
    const DeviceInfo &dev = device_info();
    if (!dev.ok || M < 1 || M > dbulk::TOK || K > dbulk::X16_MAX_K || tc::encode_fn() == nullptr) return p;
    const dbulk::Geometry geo(K);
    const long long groups = (N + dbulk::ROWS - 1) / dbulk::ROWS, sms = dev.sm_count;
    const long long xs = (long long)geo.xs_bytes(M), stage = geo.stage_bytes();
    const long long fit = ((long long)dbulk::SMEM_BUDGET - xs) / stage;
    const long long static_smem = (long long)sizeof(dbulk::Smem) + 1024;
    auto ring_for = [&](long long grid) {
        const long long items = (groups + grid - 1) / grid * geo.nst;
        long long r = items < dbulk::MAX_RING ? items : dbulk::MAX_RING;
        return r < fit ? r : fit;
    };
    auto block_smem = [&](long long ring) { return ring * stage + xs + static_smem; };
    long long grid;
    if (groups <= 2 * sms) {
        const long long per_sm = (groups + sms - 1) / sms;
        grid = 2 * per_sm * block_smem(ring_for(groups)) <= dbulk::SM_SMEM ? groups : (groups < sms ? groups : sms);
    } else {
        grid = 2 * sms;
    }
    const long long ring = ring_for(grid);
    if (ring < 1) return p;
    p.grid = (int)grid;
    p.ring_n = (int)ring;
    p.smem = (size_t)(ring * stage + xs);
    p.ok = true;
    return p;
}

template <bool EARLY, bool FUSED, int R, int J8>
cudaError_t launch_ring_kernel(const RingPlan &plan, const int8_t *Xq, int ldq, const float *sx, const float *X,
                               int ldx, int vec4, int M, int K, const uint8_t *Wp, int ldp, const float *sw, int N,
                               const float *bias, unsigned flags, void *Y, int ldy, cudaStream_t s,
                               ZpArgs zpa = ZpArgs{nullptr, nullptr}) {
    const dbulk::Geometry geo(K);
    // the packed rows as [N][kp / 8] elements of 8 bytes, stride ldp
    CUtensorMap tm_w;
    if (!tc::make_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT64, Wp, (uint64_t)(geo.kp / 8), (uint64_t)N,
                         (uint64_t)ldp, (uint32_t)(geo.sb / 8), dbulk::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = dbulk::k_decode_ring<EARLY, FUSED, R, J8>;
    if (!raise_smem_limit(reinterpret_cast<const void *>(kern), dbulk::SMEM_BUDGET)) return cudaErrorInvalidValue;
    return launch_pdl(kern, dim3(plan.grid), dim3(dbulk::THREADS), plan.smem, s, tm_w, Xq, ldq, sx, X, ldx, vec4, M,
                      K, sw, N, bias, flags, Y, ldy, plan.ring_n, zpa);
}

// Product on INT8 activations through the persistent decode kernel.
cudaError_t launch_ring_q(const RingPlan &plan, bool early, const int8_t *Xq, int ldq, const float *sx, int M,
                          int K, const uint8_t *Wp, int ldp, const float *sw, int N, const float *bias,
                          unsigned flags, void *Y, int ldy, cudaStream_t s, ZpArgs zpa) {
    if (early)
        return launch_ring_kernel<true, false, 1, 1>(plan, Xq, ldq, sx, nullptr, 0, 0, M, K, Wp, ldp, sw, N,
                                                           bias, flags, Y, ldy, s, zpa);
    return launch_ring_kernel<false, false, 1, 1>(plan, Xq, ldq, sx, nullptr, 0, 0, M, K, Wp, ldp, sw, N, bias,
                                                        flags, Y, ldy, s, zpa);
}

// Decode with the activation quantization fused in, for M <= 4: the block
// keeps R rows x J8 units of 8 floats per thread in registers when
// R * J8 <= 4 (M <= R, the stages' k <= 2048 J8), else it reads X twice.
// Every block reads all of X, so the two-pass form is taken only where that
// traffic (grid x M x K x 8 bytes) stays within the weight stream (N x K / 2
// bytes); otherwise the activation pass runs first.
int fq_rows(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }
int fq_j8(int K) {  // units per row and thread to cover the stages' k, rounded up to a power of 2
    const int j = (dbulk::Geometry(K).pitch - 16 + 2047) / 2048;
    int p = 1;
    while (p < j) p *= 2;
    return p;
}
bool fq_in_registers(int M, int K) { return fq_rows(M) * fq_j8(K) <= 4; }
bool fq_eligible(int M, int K, int N) {
    if (M > 4) return false;
    const RingPlan plan = ring_plan(M, K, N);
    return plan.ok && (fq_in_registers(M, K) || (long long)plan.grid * M * 16 <= N);
}

w4a8_status launch_fq(const float *X, int M, int K, int ldx, const uint8_t *Wp, int ldp,
                      const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                      cudaStream_t s) {
    const int vec4 = aligned16(X) && (ldx % 4 == 0);
    const RingPlan plan = ring_plan(M, K, N);
    const bool early = (flags & W4A8_STATIC_WEIGHTS) != 0;
    cudaError_t e = cudaErrorInvalidValue;
#define W4A8_FQ(E, R, J)                                                                                       \
    if (early == E && fq_rows(M) == R && fq_j8(K) == J)                                                        \
        e = launch_ring_kernel<E, true, R, J>(plan, nullptr, 0, nullptr, X, ldx, vec4, M, K, Wp, ldp, sw, N, \
                                                    bias, flags, Y, ldy, s);
    if (fq_in_registers(M, K)) {
        W4A8_FQ(true, 1, 1) W4A8_FQ(true, 1, 2) W4A8_FQ(true, 1, 4) W4A8_FQ(true, 2, 1) W4A8_FQ(true, 2, 2)
        W4A8_FQ(true, 4, 1)
        W4A8_FQ(false, 1, 1) W4A8_FQ(false, 1, 2) W4A8_FQ(false, 1, 4) W4A8_FQ(false, 2, 1) W4A8_FQ(false, 2, 2)
        W4A8_FQ(false, 4, 1)
    } else {  // J8 = 0: two passes over X
#define W4A8_FQ2(E, R)                                                                                          \
    if (early == E && fq_rows(M) == R)                                                                          \
        e = launch_ring_kernel<E, true, R, 0>(plan, nullptr, 0, nullptr, X, ldx, vec4, M, K, Wp, ldp, sw, N, bias, \
                                              flags, Y, ldy, s);
        W4A8_FQ2(true, 1) W4A8_FQ2(true, 2) W4A8_FQ2(true, 4)
        W4A8_FQ2(false, 1) W4A8_FQ2(false, 2) W4A8_FQ2(false, 4)
#undef W4A8_FQ2
    }
#undef W4A8_FQ
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    t_last_path = W4A8_PATH_DECODE;
    t_last_launches = 1;
    t_last_kernel = "k_decode_ring";
    return W4A8_OK;
}

// The cluster K-split kernel serves the chained calls (w4a8_linear_chain):
// there it replaces the activation pass and the product with one launch.
// Plain calls keep the persistent ring and the register kernel: measured on
// B200 in back-to-back launches at K = N = 4096, the split kernel's exchanges
// between the CTAs of a cluster cost more than its shorter K loop saves
// (3.98 vs 3.26 us at M = 1, 5.77 vs 4.87 us at M = 16, INT8 input).
bool split_preferred(int M, int K, int N, bool chained) {
    const dsplit::Plan pl = dsplit::plan(M, K, N);
    return chained && pl.ok && (long long)pl.nblk * pl.C <= 2LL * device_info().sm_count;
}

// On a short layer (at most two 16-channel groups per SM) whose packed rows
// are one batch of k_linear_decode<1> (K <= 4096), that kernel beats the ring
// from M = 3 rows on: each thread holds its whole share of the weights in
// registers from before the dependency wait and reads its activation
// fragments straight from L2, so neither operand makes a pass through shared
// memory after the wait (the ring stages the INT8 rows and reads every weight
// byte back from shared memory there). Measured back to back on B200 at
// K = N = 4096 with INT8 input: 3.26 vs 3.61 us at M = 4, 3.44 vs 4.46 us at
// M = 8; at M = 1 the two are level.
bool registers_beat_ring(int M, int K, int N) {
    const long long groups = (N + dbulk::ROWS - 1) / dbulk::ROWS;
    return M >= 3 && packed_row_bytes(K) <= DEC_WARPS * dec_unroll<1>() * 64 &&
           groups <= 2LL * device_info().sm_count;
}

enum DecodeKernel { DK_NONE = 0, DK_SPLIT, DK_RING, DK_REGS };

// The decode kernel for a path value of the decode family: the forced one if
// it can run the shape (DK_NONE if not), else the rule by shape.
DecodeKernel decode_kernel_for(unsigned path, int M, int K, int N, bool chained = false) {
    if (path == W4A8_PATH_DECODE_SPLIT) return dsplit::plan(M, K, N).ok ? DK_SPLIT : DK_NONE;
    if (path == W4A8_PATH_DECODE_RING) return ring_plan(M, K, N).ok ? DK_RING : DK_NONE;
    if (path == W4A8_PATH_DECODE_REGS) return DK_REGS;
    if (split_preferred(M, K, N, chained)) return DK_SPLIT;
    if (ring_plan(M, K, N).ok && !registers_beat_ring(M, K, N)) return DK_RING;
    return DK_REGS;
}

// One launch of the cluster K-split kernel. in: dsplit::IN_*; for IN_Q the
// activations are (Xq, ldq, sx), otherwise (X, ldx) with x_amax/x_parts for
// IN_F32_PARTS. y_amax: the chaining output, or null.
cudaError_t launch_split(int in, const int8_t *Xq, int ldq, const float *sx, const float *X, int ldx,
                         const float *x_amax, int x_parts, int M, int K, const uint8_t *Wp, int ldp,
                         const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                         float *y_amax, bool early, cudaStream_t s, ZpArgs zpa = ZpArgs{nullptr, nullptr}) {
    const dsplit::Plan pl = dsplit::plan(M, K, N);
    if (!pl.ok) return cudaErrorInvalidValue;
    dsplit::Params p = {};
    p.Xq = Xq;
    p.sx = sx;
    p.ldq = ldq;
    p.X = X;
    p.ldx = ldx;
    p.vec4 = X != nullptr && aligned16(X) && (ldx % 4 == 0);
    p.x_amax = x_amax;
    p.x_parts = x_parts;
    p.M = M;
    p.K = K;
    p.Wp = Wp;
    p.ldp = ldp;
    p.sw = sw;
    p.N = N;
    p.bias = bias;
    p.flags = flags;
    p.Y = Y;
    p.ldy = ldy;
    p.y_amax = y_amax;
    p.y_parts = (N + 15) / 16;
    p.ch = pl.ch;
    p.zpa = zpa;
    if (in == dsplit::IN_Q) return dsplit::launch<dsplit::IN_Q>(pl, p, early, s);
    if (in == dsplit::IN_F32) return dsplit::launch<dsplit::IN_F32>(pl, p, early, s);
    return dsplit::launch<dsplit::IN_F32_PARTS>(pl, p, early, s);
}

// act_perm: Xq uses the k-permuted layout (only the tensor-core path reads it).
// after_act_pass: the launch directly follows this library's activation pass,
// so the decode kernel may stream its weights before its dependency wait (as
// it may when the caller passes W4A8_STATIC_WEIGHTS).
// zpa: the zero-point correction of the product epilogues (null: none).
w4a8_status run_product(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                        const uint8_t *Wp, int ldp, const float *sw, int N,
                        const float *bias, unsigned flags, void *Y, int ldy,
                        cudaStream_t stream, bool act_perm = false, bool after_act_pass = false,
                        ZpArgs zpa = ZpArgs{nullptr, nullptr}) {
    const DeviceInfo &dev = device_info();
    if (!dev.ok) return W4A8_ERR_UNSUPPORTED;
    const unsigned path = choose_path(M, K, N, flags);
    const unsigned fam = path_family(path);
    if (act_perm && fam != W4A8_PATH_TC) return W4A8_ERR_INVALID_ARG;
    const DecodeKernel dk = fam == W4A8_PATH_DECODE ? decode_kernel_for(path, M, K, N) : DK_NONE;
    if (fam == W4A8_PATH_DECODE && dk == DK_NONE) return W4A8_ERR_UNSUPPORTED;
    const bool early = after_act_pass || (flags & W4A8_STATIC_WEIGHTS);
    cudaError_t e = cudaSuccess;
    const char *kernel = "";
    if (fam == W4A8_PATH_GENERIC) {
        kernel = "k_linear_generic";
        dim3 grid((N + 127) / 128, (unsigned)(M < 65535 ? M : 65535));
        e = launch_pdl(k_linear_generic, grid, dim3(128), 0, stream,
                       Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, zpa);
    } else if (dk == DK_SPLIT) {
        kernel = "k_decode_split";
        e = launch_split(dsplit::IN_Q, Xq, ldq, sx, nullptr, 0, nullptr, 0, M, K, Wp, ldp, sw, N, bias, flags, Y,
                         ldy, nullptr, early, stream, zpa);
    } else if (dk == DK_RING) {
        kernel = "k_decode_ring";
        e = launch_ring_q(ring_plan(M, K, N), early, Xq, ldq, sx, M, K, Wp, ldp, sw, N, bias, flags, Y, ldy, stream,
                          zpa);
    } else if (dk == DK_REGS) {
        kernel = "k_linear_decode";
        const int tok = M <= 8 ? 8 : 16;
        const int tiles = (M + tok - 1) / tok;
        if (tiles > 65535) return W4A8_ERR_UNSUPPORTED;
        dim3 grid((N + 15) / 16, tiles);
        auto kern = tok == 8 ? (early ? k_linear_decode<1, true> : k_linear_decode<1, false>)
                             : (early ? k_linear_decode<2, true> : k_linear_decode<2, false>);
        e = launch_pdl(kern, grid, dim3(DEC_WARPS * 32), 0, stream,
                       Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, zpa);
    } else if (fam == W4A8_PATH_TC) {
        if (!tc_supported(M, K, N)) return W4A8_ERR_UNSUPPORTED;
        w4a8_status st;
        const bool forced = (flags & W4A8_PATH_MASK) != 0;
        if (path == W4A8_PATH_TC_PAIR || (!forced && pair_preferred(M, K, N))) {
            kernel = "k_gemm_tc_pair";
            if (K > tc::TC_X16_MAX_K) return W4A8_ERR_UNSUPPORTED;
            st = act_perm ? tcp::launch<tc::UNPACK_X16_PERM>(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy,
                                                             dev.sm_count, stream, zpa)
                          : tcp::launch<tc::UNPACK_X16>(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy,
                                                        dev.sm_count, stream, zpa);
        } else {
            kernel = "k_gemm_tc";
            st = launch_gemm_tc(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy, dev.sm_count, stream,
                                act_perm, zpa);
        }
        if (st != W4A8_OK) return st;
    } else {
        return W4A8_ERR_INVALID_ARG;
    }
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    t_last_path = fam;
    t_last_launches = 1;
    t_last_kernel = kernel;
    return W4A8_OK;
}

// -------------------------------------------------------- zero-point INT4 ---
// Workspace of the zero-point calls: the INT8 rows and scales (w4z_linear
// only), the row sums of the INT8 rows, and the INT32 accumulators of the
// unchanged W4A8 product on the q - 8 codes.
struct ZWorkspace {
    Workspace a;
    int *rowsum;
};

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

size_t zworkspace_bytes(int M, int K, int N) {
    (void)N;
    const int ldq = round_up(K, 16);
    return round256((size_t)M * (size_t)ldq) + 2 * round256(sizeof(float) * (size_t)M) + 256;
}

ZWorkspace carve_zworkspace(void *ws, int M, int K) {
    ZWorkspace z;
    z.a = carve_workspace(ws, M, K);
    uintptr_t p = reinterpret_cast<uintptr_t>(z.a.sx) + round256(sizeof(float) * (size_t)M);
    z.rowsum = reinterpret_cast<int *>(p);
    return z;
}

// The zero-point product on INT8 rows: the row sums (unless the activation
// pass already wrote them), then the W4A8 product on the q - 8 codes with the
// correction acc' - (zp - 8) * rowsum in its epilogue. after_act_pass: as for
// run_product.
w4a8_status run_product_z(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                          const float *sa, const int32_t *zp, int N, const float *bias, unsigned flags, void *Y,
                          int ldy, const ZWorkspace &zw, cudaStream_t s, bool after_act_pass, bool act_perm,
                          bool have_rowsum) {
    if (!have_rowsum) {
        const int rows = M < 65535 ? M : 65535;
        cudaError_t e = launch_pdl(zpt::k_row_sum8, dim3(rows), dim3(256), 0, s, Xq, M, K, ldq, zw.rowsum);
        if (e != cudaSuccess) return W4A8_ERR_CUDA;
        // the row-sum kernel waits before it lets dependents start, so the
        // product may treat the weights as final exactly as behind the activation pass
        after_act_pass = true;
    }
    return run_product(Xq, M, K, ldq, sx, Wp, ldp, sa, N, bias, flags, Y, ldy, s, act_perm, after_act_pass,
                       ZpArgs{zp, zw.rowsum});
}

// ------------------------------------------------------- group-wise INT4 ---
// The group-wise product (any M, tiles of 8 or 16 tokens; float32 outputs).
// The group-wise path: the tensor-core form for many rows (or W4A8_PATH_TC),
// the decode-style kernel for few rows (or the decode family forced).
unsigned path_g(int M, unsigned flags) {
    const unsigned path = flags & W4A8_PATH_MASK;
    if (path == W4A8_PATH_TC) return W4A8_PATH_TC;
    if (path != W4A8_PATH_AUTO && path_family(path) != W4A8_PATH_DECODE) return 0;
    if (path == W4A8_PATH_AUTO && M > 16 && tc::encode_fn() != nullptr) return W4A8_PATH_TC;
    return W4A8_PATH_DECODE;
}

// act_perm: Xq uses the k-permuted layout (only the tensor-core form reads it).
w4a8_status run_product_g(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                          const float *sa, const int32_t *zp, int N, const float *bias, unsigned flags, void *Y,
                          int ldy, cudaStream_t stream, bool after_act_pass, bool act_perm = false) {
    const unsigned path = path_g(M, flags);
    if (path == 0) return W4A8_ERR_UNSUPPORTED;
    if (path == W4A8_PATH_TC) {
        if (!tc_supported(M, K, N)) return W4A8_ERR_UNSUPPORTED;
        const int sms = device_info().sm_count;
        w4a8_status st = act_perm ? tcg::launch<true>(Xq, M, K, ldq, sx, Wp, ldp, sa, zp, grp::groups_of(K), N, bias,
                                                      flags, Y, ldy, sms, stream)
                                  : tcg::launch<false>(Xq, M, K, ldq, sx, Wp, ldp, sa, zp, grp::groups_of(K), N, bias,
                                                       flags, Y, ldy, sms, stream);
        if (st != W4A8_OK) return st;
        t_last_path = W4A8_PATH_TC;
        t_last_launches = 1;
        t_last_kernel = "k_gemm_tc_grp";
        return W4A8_OK;
    }
    if (act_perm) return W4A8_ERR_INVALID_ARG;
    const int tok = M <= 8 ? 8 : 16;
    const int tiles = (M + tok - 1) / tok;
    if (tiles > 65535) return W4A8_ERR_UNSUPPORTED;
    dim3 grid((N + 15) / 16, tiles);
    const bool early = after_act_pass || (flags & W4A8_STATIC_WEIGHTS);
    auto kern = tok == 8 ? (early ? grp::k_linear_g<1, true> : grp::k_linear_g<1, false>)
                         : (early ? grp::k_linear_g<2, true> : grp::k_linear_g<2, false>);
    cudaError_t e = launch_pdl(kern, grid, dim3(DEC_WARPS * 32), 0, stream, Xq, M, K, ldq, sx, Wp, ldp, sa, zp,
                               grp::groups_of(K), N, bias, flags, Y, ldy);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    t_last_path = W4A8_PATH_DECODE;
    t_last_launches = 1;
    t_last_kernel = "k_linear_g";
    return W4A8_OK;
}

// ------------------------------------------------------------------ W8A8 ---
// The INT8 path the INT4 steps extend: one INT8 weight code per byte, rows
// of ldw8 >= K bytes (a multiple of 16), the same argument rules otherwise.
w4a8_status check_common8(int M, int K, int N, const int8_t *Wq, int ldw8, const float *sw,
                          const float *bias, unsigned flags, const void *Y, int ldy) {
    if (K < 1 || K > W8A8_MAX_K || N < 1 || M < 0) return W4A8_ERR_INVALID_ARG;
    if (!Wq || !aligned16(Wq) || ldw8 < K || ldw8 % 16 != 0) return W4A8_ERR_INVALID_ARG;
    // the remaining rules are the INT4 layer's (its row check passes for ldw8)
    return check_common(M, K, N, reinterpret_cast<const uint8_t *>(Wq), ldw8, sw, bias, flags, Y, ldy);
}

// The W8A8 product on INT8 activations (natural k order).
w4a8_status run_product8(const int8_t *Xq, int M, int K, int ldq, const float *sx, const int8_t *Wq, int ldw8,
                         const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                         cudaStream_t stream, bool after_act_pass = false) {
    const DeviceInfo &dev = device_info();
    if (!dev.ok) return W4A8_ERR_UNSUPPORTED;
    if ((flags & W4A8_PATH_MASK) == W4A8_PATH_TC_PAIR) return W4A8_ERR_UNSUPPORTED;  // INT4 codes only
    const unsigned path = path_family(choose_path(M, K, N, flags));
    cudaError_t e = cudaSuccess;
    const char *kernel = "";
    if (path == W4A8_PATH_GENERIC) {
        kernel = "k_linear8_generic";
        dim3 grid((N + 127) / 128, (unsigned)(M < 65535 ? M : 65535));
        e = launch_pdl(k_linear8_generic, grid, dim3(128), 0, stream, Xq, M, K, ldq, sx, Wq, ldw8, sw, N, bias,
                       flags, Y, ldy);
    } else if (path == W4A8_PATH_DECODE) {
        kernel = "k_linear8_decode";
        const int tok = M <= 8 ? 8 : 16;
        const int tiles = (M + tok - 1) / tok;
        if (tiles > 65535) return W4A8_ERR_UNSUPPORTED;
        dim3 grid((N + 15) / 16, tiles);
        const bool early = after_act_pass || (flags & W4A8_STATIC_WEIGHTS);
        auto kern = tok == 8 ? (early ? k_linear8_decode<1, true> : k_linear8_decode<1, false>)
                             : (early ? k_linear8_decode<2, true> : k_linear8_decode<2, false>);
        e = launch_pdl(kern, grid, dim3(DEC_WARPS * 32), 0, stream, Xq, M, K, ldq, sx, Wq, ldw8, sw, N, bias, flags,
                       Y, ldy);
    } else if (path == W4A8_PATH_TC) {
        kernel = "k_gemm_tc";
        if (!tc_supported(M, K, N)) return W4A8_ERR_UNSUPPORTED;
        w4a8_status st = launch_gemm_tc8(Xq, M, K, ldq, sx, Wq, ldw8, sw, N, bias, flags, Y, ldy, dev.sm_count,
                                         stream);
        if (st != W4A8_OK) return st;
    } else {
        return W4A8_ERR_INVALID_ARG;
    }
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    t_last_path = path;
    t_last_launches = 1;
    t_last_kernel = kernel;
    return W4A8_OK;
}

// One launch of the grouped decode kernel over probs[0..count) (count <= 64,
// every M >= 1).
template <bool EARLY, int R>
cudaError_t launch_grouped_kernel(const dbulk::GroupedTable &tab, int grid, int ring_n, size_t smem, unsigned flags,
                                  cudaStream_t s) {
    auto kern = dbulk::k_decode_grouped<EARLY, R>;
    if (!raise_smem_limit(reinterpret_cast<const void *>(kern), dbulk::SMEM_BUDGET)) return cudaErrorInvalidValue;
    return launch_pdl(kern, dim3(grid), dim3(dbulk::THREADS), smem, s, tab, flags, ring_n);
}

w4a8_status launch_grouped_chunk(const w4a8_problem *probs, int count, unsigned flags, cudaStream_t s) {
    static dbulk::GroupedTable tab;  // built under the lock, copied into the launch parameters
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    memset(&tab, 0, sizeof(tab));
    int total = 0, max_m = 0, max_pitch = 0;
    long long total_bytes = 0;
    for (int i = 0; i < count; ++i) {
        const w4a8_problem &p = probs[i];
        const dbulk::Geometry geo(p.K);
        dbulk::GroupedProblem &q = tab.p[i];
        if (!tc::make_map_2d(&q.tm, CU_TENSOR_MAP_DATA_TYPE_UINT64, p.Wp, (uint64_t)(geo.kp / 8), (uint64_t)p.N,
                             (uint64_t)p.ldp, (uint32_t)(geo.sb / 8), dbulk::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
            return W4A8_ERR_CUDA;
        q.X = p.X;
        q.sw = p.sw;
        q.bias = p.bias;
        q.Y = p.Y;
        q.M = p.M;
        q.K = p.K;
        q.ldx = p.ldx;
        q.ldy = p.ldy;
        q.N = p.N;
        q.vec4 = aligned16(p.X) && (p.ldx % 4 == 0);
        q.group0 = total;
        q.bytes0 = total_bytes;
        q.group_bytes = (long long)dbulk::ROWS * geo.kp;
        total += (p.N + dbulk::ROWS - 1) / dbulk::ROWS;
        total_bytes += q.group_bytes * ((p.N + dbulk::ROWS - 1) / dbulk::ROWS);
        max_m = max_m > p.M ? max_m : p.M;
        max_pitch = max_pitch > geo.pitch ? max_pitch : geo.pitch;
    }
    tab.count = count;
    tab.total_groups = total;
    tab.total_bytes = total_bytes;
    const int r = fq_rows(max_m);
    const long long xs = (long long)r * max_pitch;
    const long long ring = ((long long)dbulk::SMEM_BUDGET - xs) / dbulk::GROUPED_SLOT;
    if (ring < 1) return W4A8_ERR_UNSUPPORTED;
    const int ring_n = (int)(ring < dbulk::MAX_RING ? ring : dbulk::MAX_RING);
    const int sms = device_info().sm_count;
    const int grid = total < 2 * sms ? total : 2 * sms;
    const size_t smem = (size_t)ring_n * dbulk::GROUPED_SLOT + (size_t)xs;
    const bool early = (flags & W4A8_STATIC_WEIGHTS) != 0;
    cudaError_t e;
    if (r == 1)
        e = early ? launch_grouped_kernel<true, 1>(tab, grid, ring_n, smem, flags, s)
                  : launch_grouped_kernel<false, 1>(tab, grid, ring_n, smem, flags, s);
    else if (r == 2)
        e = early ? launch_grouped_kernel<true, 2>(tab, grid, ring_n, smem, flags, s)
                  : launch_grouped_kernel<false, 2>(tab, grid, ring_n, smem, flags, s);
    else
        e = early ? launch_grouped_kernel<true, 4>(tab, grid, ring_n, smem, flags, s)
                  : launch_grouped_kernel<false, 4>(tab, grid, ring_n, smem, flags, s);
    return from_cuda(e);
}

// Self-test of the failure path: one thread waits on an mbarrier that no one
// arrives on; the bounded wait gives up after `limit` cycles, records
// W4A8_ERR_TIMEOUT in the device status word and the kernel returns.
__global__ void k_selftest_timeout(long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)ptx::mbar_wait(&bar, 0, &abort_flag, limit);
}

// Scratch of w4a8_linear_noalloc: a file-scope device array, so callers that
// cannot allocate still get somewhere to keep the INT8 activations.
static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A8_NOALLOC_SCRATCH_BYTES];

// The array's device address, looked up once per device with that device
// current. In host code the symbol g_noalloc_scratch is only a host-side
// stand-in and must never be handed to a kernel.
void *noalloc_scratch_ptr() {
    static std::mutex mu;
    static void *ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = p;
    }
    return ptrs[dev];
}

}  // namespace
}  // namespace w4a8

using namespace w4a8;

extern "C" {

int w4a8_packed_ld(int K) { return K < 1 ? -1 : round_up((K + 1) / 2, 16); }

int w4a8_act_ld(int K) { return K < 1 ? -1 : round_up(K, 16); }

size_t w4a8_workspace_size(int M, int K) {
    if (M < 0 || K < 1) return 0;
    return workspace_bytes_for(M, K, nullptr);
}

w4a8_status w4_quantize_pack(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp,
                             float *sw, void *stream) {
    if (!W || !Wp || !sw || K < 1 || K > W4A8_MAX_K || N < 1 || ldw < N) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(Wp) || ldp < (K + 1) / 2 || ldp % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (!aligned4(W) || !aligned4(sw)) return W4A8_ERR_INVALID_ARG;
    const DeviceInfo &dev = device_info();
    if (!dev.ok) return W4A8_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // One pass over W (cluster panels in shared memory) where TMA can tile
    // the layout and a slice fits; the two-pass form otherwise.
    if (qpp::eligible(W, K, ldw)) return qpp::launch<4>(W, K, N, ldw, Wp, ldp, sw, s);
    unsigned *amax = reinterpret_cast<unsigned *>(sw);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * (size_t)N, s);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    // VEC = 4 (float4 rows) when the layout allows it.
    const bool v4 = (N % 4 == 0) && (ldw % 4 == 0) && aligned16(W);
    const int cols = v4 ? 128 : 32;
    const int col_blocks = (N + cols - 1) / cols;
    // K-slices so that the abs-max pass puts several blocks on every SM.
    int splits = (6 * dev.sm_count + col_blocks - 1) / col_blocks;
    splits = splits < 1 ? 1 : splits;
    int rows = (K + splits - 1) / splits;
    rows = round_up(rows < 64 ? 64 : rows, 32);
    splits = (K + rows - 1) / rows;
    if (splits > 65535) return W4A8_ERR_UNSUPPORTED;
    if (v4)
        k_col_absmax<4><<<dim3(col_blocks, splits), 256, 0, s>>>(W, K, N, ldw, rows, amax);
    else
        k_col_absmax<1><<<dim3(col_blocks, splits), 256, 0, s>>>(W, K, N, ldw, rows, amax);
    if ((e = cudaGetLastError()) != cudaSuccess) return W4A8_ERR_CUDA;
    const int kblocks = (2 * ldp + 63) / 64;
    if (kblocks > 65535) return W4A8_ERR_UNSUPPORTED;
    if (v4)
        k_quant_pack<4><<<dim3(col_blocks, kblocks), 256, 0, s>>>(W, K, N, ldw, amax, Wp, ldp);
    else
        k_quant_pack<1><<<dim3(col_blocks, kblocks), 256, 0, s>>>(W, K, N, ldw, amax, Wp, ldp);
    if ((e = cudaGetLastError()) != cudaSuccess) return W4A8_ERR_CUDA;
    k_weight_scale_finalize<7><<<(N + 255) / 256, 256, 0, s>>>(sw, N);
    return from_cuda(cudaGetLastError());
}

int w8a8_ld(int K) { return K < 1 ? -1 : round_up(K, 16); }

int w4g_groups(int K) { return K < 1 ? -1 : grp::groups_of(K); }

w4a8_status w4g_quantize_pack(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp, float *sa, int32_t *zp,
                              void *stream) {
    if (!W || !Wp || !sa || !zp || K < 1 || K > W4A8_MAX_K || N < 1 || ldw < N) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(Wp) || ldp < (K + 1) / 2 || ldp % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (!aligned4(W) || !aligned4(sa) || !aligned4(zp)) return W4A8_ERR_INVALID_ARG;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // every byte of every row, the parts no group covers included, starts at 0
    cudaError_t e = cudaMemset2DAsync(Wp, (size_t)ldp, 0, (size_t)ldp, (size_t)N, s);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    const int ng = grp::groups_of(K);
    grp::k_quant_pack_g<<<dim3((N + 127) / 128, ng), 128, 0, s>>>(W, K, N, ldw, Wp, ldp, sa, zp, ng);
    return from_cuda(cudaGetLastError());
}

size_t w4z_workspace_size(int M, int K, int N) {
    if (M < 0 || K < 1 || N < 1) return 0;
    return zworkspace_bytes(M, K, N);
}

w4a8_status w4z_quantize_pack(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp, float *sa, int32_t *zp,
                              void *stream) {
    if (!W || !Wp || !sa || !zp || K < 1 || K > W4A8_MAX_K || N < 1 || ldw < N) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(Wp) || ldp < (K + 1) / 2 || ldp % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (!aligned4(W) || !aligned4(sa) || !aligned4(zp)) return W4A8_ERR_INVALID_ARG;
    const DeviceInfo &dev = device_info();
    if (!dev.ok) return W4A8_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int *lo = reinterpret_cast<int *>(zp), *hi = reinterpret_cast<int *>(sa);
    zpt::k_minmax_init<<<(N + 255) / 256, 256, 0, s>>>(lo, hi, N);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    const int col_blocks = (N + 31) / 32;
    int splits = (6 * dev.sm_count + col_blocks - 1) / col_blocks;
    splits = splits < 1 ? 1 : splits;
    int rows = (K + splits - 1) / splits;
    rows = rows < 64 ? 64 : rows;
    splits = (K + rows - 1) / rows;
    if (splits > 65535) return W4A8_ERR_UNSUPPORTED;
    zpt::k_col_minmax<<<dim3(col_blocks, splits), 256, 0, s>>>(W, K, N, ldw, rows, lo, hi);
    if ((e = cudaGetLastError()) != cudaSuccess) return W4A8_ERR_CUDA;
    zpt::k_zp_finalize<<<(N + 255) / 256, 256, 0, s>>>(lo, hi, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return W4A8_ERR_CUDA;
    const int kblocks = (2 * ldp + 63) / 64;
    if (kblocks > 65535) return W4A8_ERR_UNSUPPORTED;
    zpt::k_quant_pack_z<<<dim3(col_blocks, kblocks), 256, 0, s>>>(W, K, N, ldw, sa, zp, Wp, ldp);
    return from_cuda(cudaGetLastError());
}

w4a8_status w8_quantize(const float *W, int K, int N, int ldw, int8_t *Wq, int ldw8, float *sw, void *stream) {
    if (!W || !Wq || !sw || K < 1 || K > W8A8_MAX_K || N < 1 || ldw < N) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(Wq) || ldw8 < K || ldw8 % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (!aligned4(W) || !aligned4(sw)) return W4A8_ERR_INVALID_ARG;
    const DeviceInfo &dev = device_info();
    if (!dev.ok) return W4A8_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // one pass over W where the layout allows it, as for the INT4 weights
    if (qpp::eligible(W, K, ldw))
        return qpp::launch<8>(W, K, N, ldw, reinterpret_cast<uint8_t *>(Wq), ldw8, sw, s);
    unsigned *amax = reinterpret_cast<unsigned *>(sw);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * (size_t)N, s);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    const bool v4 = (N % 4 == 0) && (ldw % 4 == 0) && aligned16(W);
    const int cols = v4 ? 128 : 32;
    const int col_blocks = (N + cols - 1) / cols;
    int splits = (6 * dev.sm_count + col_blocks - 1) / col_blocks;
    splits = splits < 1 ? 1 : splits;
    int rows = (K + splits - 1) / splits;
    rows = round_up(rows < 64 ? 64 : rows, 32);
    splits = (K + rows - 1) / rows;
    if (splits > 65535) return W4A8_ERR_UNSUPPORTED;
    if (v4)
        k_col_absmax<4><<<dim3(col_blocks, splits), 256, 0, s>>>(W, K, N, ldw, rows, amax);
    else
        k_col_absmax<1><<<dim3(col_blocks, splits), 256, 0, s>>>(W, K, N, ldw, rows, amax);
    if ((e = cudaGetLastError()) != cudaSuccess) return W4A8_ERR_CUDA;
    const int kblocks = (ldw8 + 31) / 32;
    if (kblocks > 65535) return W4A8_ERR_UNSUPPORTED;
    if (v4)
        k_quant8<4><<<dim3(col_blocks, kblocks), 256, 0, s>>>(W, K, N, ldw, amax, Wq, ldw8);
    else
        k_quant8<1><<<dim3(col_blocks, kblocks), 256, 0, s>>>(W, K, N, ldw, amax, Wq, ldw8);
    if ((e = cudaGetLastError()) != cudaSuccess) return W4A8_ERR_CUDA;
    k_weight_scale_finalize<127><<<(N + 255) / 256, 256, 0, s>>>(sw, N);
    return from_cuda(cudaGetLastError());
}

// rowsum: also write sum_k xq[m][k] per row (the zero-point form), or null.
static w4a8_status launch_act_quant(const float *X, int M, int K, int ldx, int8_t *Xq, int ldq,
                                    float *sx, cudaStream_t s, bool perm = false, int32_t *rowsum = nullptr) {
    const int vec4 = aligned16(X) && (ldx % 4 == 0);
    const int grid = M < 65535 ? M : 65535;
    cudaError_t e;
    // One block per row. With few rows (fewer than two per SM) a long row
    // gets a 1024-thread block that holds it in registers up to K = 32768;
    // many rows keep 256-thread blocks, several per SM, and read a long row
    // twice.
    const bool wide = K > 4096 && M < 2 * device_info().sm_count;
    if (perm) {
        if (K <= 1024)
            e = launch_pdl(k_act_quant<128, 8, true>, dim3(grid), dim3(128), 0, s,
                           X, M, K, ldx, Xq, ldq, sx, vec4, rowsum);
        else if (!wide)
            e = launch_pdl(k_act_quant<256, 16, true>, dim3(grid), dim3(256), 0, s,
                           X, M, K, ldx, Xq, ldq, sx, vec4, rowsum);
        else
            e = launch_pdl(k_act_quant<1024, 32, true>, dim3(grid), dim3(1024), 0, s,
                           X, M, K, ldx, Xq, ldq, sx, vec4, rowsum);
    } else {
        if (K <= 1024)
            e = launch_pdl(k_act_quant<128, 8, false>, dim3(grid), dim3(128), 0, s,
                           X, M, K, ldx, Xq, ldq, sx, vec4, rowsum);
        else if (!wide)
            e = launch_pdl(k_act_quant<256, 16, false>, dim3(grid), dim3(256), 0, s,
                           X, M, K, ldx, Xq, ldq, sx, vec4, rowsum);
        else
            e = launch_pdl(k_act_quant<1024, 32, false>, dim3(grid), dim3(1024), 0, s, X, M, K, ldx, Xq, ldq, sx,
                           vec4, rowsum);
    }
    return from_cuda(e);
}

// Steps 3-6 on float32 activations with the INT8 copy in `ws`: the path is
// chosen first, so the tensor-core GEMM gets its k-permuted activation layout
// and a few-row decode quantizes inside its own kernel.
static w4a8_status linear_from_f32(const float *X, int M, int K, int ldx, const uint8_t *Wp, int ldp,
                                   const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                                   const Workspace &ws, cudaStream_t s) {
    const unsigned path = choose_path(M, K, N, flags);
    const unsigned fam = path_family(path);
    const DecodeKernel dk = fam == W4A8_PATH_DECODE ? decode_kernel_for(path, M, K, N) : DK_NONE;
    if (fam == W4A8_PATH_DECODE && dk == DK_NONE) return W4A8_ERR_UNSUPPORTED;
    if (dk == DK_SPLIT) {
        // one launch: the K-split kernel quantizes its slices itself
        cudaError_t e = launch_split(dsplit::IN_F32, nullptr, 0, nullptr, X, ldx, nullptr, 0, M, K, Wp, ldp, sw, N,
                                     bias, flags, Y, ldy, nullptr, (flags & W4A8_STATIC_WEIGHTS) != 0, s);
        if (e != cudaSuccess) return W4A8_ERR_CUDA;
        t_last_path = W4A8_PATH_DECODE;
        t_last_launches = 1;
        t_last_kernel = "k_decode_split";
        return W4A8_OK;
    }
    if (dk == DK_RING && fq_eligible(M, K, N)) return launch_fq(X, M, K, ldx, Wp, ldp, sw, N, bias, flags, Y, ldy, s);
    const bool perm = fam == W4A8_PATH_TC && K <= tc::TC_X16_MAX_K;
    w4a8_status st = launch_act_quant(X, M, K, ldx, ws.xq, ws.ldq, ws.sx, s, perm);
    if (st != W4A8_OK) return st;
    st = run_product(ws.xq, M, K, ws.ldq, ws.sx, Wp, ldp, sw, N, bias, flags, Y, ldy, s, perm, true);
    if (st == W4A8_OK) t_last_launches = 2;
    return st;
}

w4a8_status a8_quantize_rows(const float *X, int M, int K, int ldx, int8_t *Xq, int ldq,
                             float *sx, void *stream) {
    if (M < 0 || K < 1 || K > W4A8_MAX_K || ldx < K) return W4A8_ERR_INVALID_ARG;
    if (ldq < K || ldq % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!X || !Xq || !sx || !aligned16(Xq) || !aligned4(X) || !aligned4(sx)) return W4A8_ERR_INVALID_ARG;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    return launch_act_quant(X, M, K, ldx, Xq, ldq, sx, static_cast<cudaStream_t>(stream));
}

w4a8_status w4a8_linear(const float *X, int M, int K, int ldx, const uint8_t *Wp, int ldp,
                        const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                        void *workspace, size_t workspace_bytes, void *stream) {
    w4a8_status st = check_common(M, K, N, Wp, ldp, sw, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldx < K) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!X || !aligned4(X)) return W4A8_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    if (workspace_bytes < w4a8_workspace_size(M, K)) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    const Workspace ws = carve_workspace(workspace, M, K);
    return linear_from_f32(X, M, K, ldx, Wp, ldp, sw, N, bias, flags, Y, ldy, ws,
                           static_cast<cudaStream_t>(stream));
}

w4a8_status w4a8_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                          const uint8_t *Wp, int ldp, const float *sw, int N, const float *bias,
                          unsigned flags, void *Y, int ldy, void *stream) {
    w4a8_status st = check_common(M, K, N, Wp, ldp, sw, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldq < K || ldq % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!Xq || !sx || !aligned16(Xq) || !aligned4(sx)) return W4A8_ERR_INVALID_ARG;
    return run_product(Xq, M, K, ldq, sx, Wp, ldp, sw, N, bias, flags, Y, ldy,
                       static_cast<cudaStream_t>(stream));
}

w4a8_status w4a8_linear_noalloc(const float *X, int M, int K, int ldx, const uint8_t *Wp, int ldp,
                                const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                                void *stream) {
    w4a8_status st = check_common(M, K, N, Wp, ldp, sw, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldx < K) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!X || !aligned4(X)) return W4A8_ERR_INVALID_ARG;
    if (w4a8_workspace_size(M, K) > (size_t)W4A8_NOALLOC_SCRATCH_BYTES) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    void *scratch = noalloc_scratch_ptr();
    if (!scratch) return W4A8_ERR_CUDA;
    const Workspace ws = carve_workspace(scratch, M, K);
    return linear_from_f32(X, M, K, ldx, Wp, ldp, sw, N, bias, flags, Y, ldy, ws,
                           static_cast<cudaStream_t>(stream));
}

size_t w4a8_noalloc_scratch_bytes(void) { return (size_t)W4A8_NOALLOC_SCRATCH_BYTES; }

int w4a8_amax_parts(int N) { return N < 1 ? -1 : (N + 15) / 16; }

w4a8_status w4a8_linear_chain(const float *X, int M, int K, int ldx, const float *x_amax, int x_parts,
                              const uint8_t *Wp, int ldp, const float *sw, int N, const float *bias, unsigned flags,
                              float *Y, int ldy, float *y_amax, void *workspace, size_t workspace_bytes,
                              void *stream) {
    if ((flags & W4A8_OUT_MASK) != W4A8_OUT_F32) return W4A8_ERR_INVALID_ARG;
    w4a8_status st = check_common(M, K, N, Wp, ldp, sw, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldx < K) return W4A8_ERR_INVALID_ARG;
    if (x_amax && (x_parts < 1 || !aligned4(x_amax))) return W4A8_ERR_INVALID_ARG;
    if (y_amax && !aligned4(y_amax)) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!X || !aligned4(X)) return W4A8_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    if (workspace_bytes < w4a8_workspace_size(M, K)) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned path = choose_path(M, K, N, flags);
    const unsigned fam = path_family(path);
    const int y_parts = (N + 15) / 16;
    if (fam == W4A8_PATH_GENERIC) {
        dim3 grid((N + chain::GEN_THREADS - 1) / chain::GEN_THREADS, (unsigned)(M < 65535 ? M : 65535));
        cudaError_t e = launch_pdl(chain::k_linear_generic_f32, grid, dim3(chain::GEN_THREADS), 0, s, X, M, K, ldx,
                                   x_amax, x_parts, Wp, ldp, sw, N, bias, flags, Y, ldy, y_amax, y_parts);
        if (e != cudaSuccess) return W4A8_ERR_CUDA;
        t_last_path = W4A8_PATH_GENERIC;
        t_last_launches = 1;
        t_last_kernel = "k_linear_generic";
        return W4A8_OK;
    }
    const DecodeKernel dk = fam == W4A8_PATH_DECODE ? decode_kernel_for(path, M, K, N, true) : DK_NONE;
    if (fam == W4A8_PATH_DECODE && dk == DK_NONE) return W4A8_ERR_UNSUPPORTED;
    if (dk == DK_SPLIT) {
        cudaError_t e = launch_split(x_amax ? dsplit::IN_F32_PARTS : dsplit::IN_F32, nullptr, 0, nullptr, X, ldx,
                                     x_amax, x_parts, M, K, Wp, ldp, sw, N, bias, flags, Y, ldy, y_amax,
                                     (flags & W4A8_STATIC_WEIGHTS) != 0, s);
        if (e != cudaSuccess) return W4A8_ERR_CUDA;
        t_last_path = W4A8_PATH_DECODE;
        t_last_launches = 1;
        t_last_kernel = "k_decode_split";
        return W4A8_OK;
    }
    // the other kernels: the activation pass and the product, then the parts
    const Workspace ws = carve_workspace(workspace, M, K);
    st = linear_from_f32(X, M, K, ldx, Wp, ldp, sw, N, bias, flags, Y, ldy, ws, s);
    if (st != W4A8_OK || !y_amax) return st;
    const unsigned launches = t_last_launches;
    dim3 grid((y_parts + 127) / 128, (unsigned)(M < 65535 ? M : 65535));
    cudaError_t e = launch_pdl(chain::k_row_amax_parts, grid, dim3(128), 0, s, static_cast<const float *>(Y), M, N,
                               ldy, y_amax, y_parts);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
    t_last_launches = launches + 1;
    return W4A8_OK;
}

w4a8_status w8a8_linear(const float *X, int M, int K, int ldx, const int8_t *Wq, int ldw8,
                        const float *sw, int N, const float *bias, unsigned flags, void *Y, int ldy,
                        void *workspace, size_t workspace_bytes, void *stream) {
    w4a8_status st = check_common8(M, K, N, Wq, ldw8, sw, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldx < K) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!X || !aligned4(X)) return W4A8_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    if (workspace_bytes < w4a8_workspace_size(M, K)) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    const Workspace ws = carve_workspace(workspace, M, K);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_act_quant(X, M, K, ldx, ws.xq, ws.ldq, ws.sx, s);
    if (st != W4A8_OK) return st;
    st = run_product8(ws.xq, M, K, ws.ldq, ws.sx, Wq, ldw8, sw, N, bias, flags, Y, ldy, s, true);
    if (st == W4A8_OK) t_last_launches = 2;
    return st;
}

w4a8_status w8a8_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                          const int8_t *Wq, int ldw8, const float *sw, int N, const float *bias,
                          unsigned flags, void *Y, int ldy, void *stream) {
    w4a8_status st = check_common8(M, K, N, Wq, ldw8, sw, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldq < K || ldq % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!Xq || !sx || !aligned16(Xq) || !aligned4(sx)) return W4A8_ERR_INVALID_ARG;
    return run_product8(Xq, M, K, ldq, sx, Wq, ldw8, sw, N, bias, flags, Y, ldy,
                        static_cast<cudaStream_t>(stream));
}

w4a8_status w4z_linear(const float *X, int M, int K, int ldx, const uint8_t *Wp, int ldp, const float *sa,
                       const int32_t *zp, int N, const float *bias, unsigned flags, void *Y, int ldy,
                       void *workspace, size_t workspace_bytes, void *stream) {
    w4a8_status st = check_common(M, K, N, Wp, ldp, sa, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (!zp || !aligned4(zp) || ldx < K) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!X || !aligned4(X)) return W4A8_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    if (workspace_bytes < w4z_workspace_size(M, K, N)) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    const ZWorkspace zw = carve_zworkspace(workspace, M, K);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the activation pass writes the row sums too; the tensor-core product
    // reads its k-permuted layout
    const bool perm = path_family(choose_path(M, K, N, flags)) == W4A8_PATH_TC && K <= tc::TC_X16_MAX_K;
    st = launch_act_quant(X, M, K, ldx, zw.a.xq, zw.a.ldq, zw.a.sx, s, perm, zw.rowsum);
    if (st != W4A8_OK) return st;
    st = run_product_z(zw.a.xq, M, K, zw.a.ldq, zw.a.sx, Wp, ldp, sa, zp, N, bias, flags, Y, ldy, zw, s, true, perm,
                       true);
    if (st == W4A8_OK) t_last_launches = 2;
    return st;
}

w4a8_status w4z_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                         const float *sa, const int32_t *zp, int N, const float *bias, unsigned flags, void *Y,
                         int ldy, void *workspace, size_t workspace_bytes, void *stream) {
    w4a8_status st = check_common(M, K, N, Wp, ldp, sa, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (!zp || !aligned4(zp) || ldq < K || ldq % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!Xq || !sx || !aligned16(Xq) || !aligned4(sx)) return W4A8_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    if (workspace_bytes < w4z_workspace_size(M, K, N)) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    const ZWorkspace zw = carve_zworkspace(workspace, M, K);
    st = run_product_z(Xq, M, K, ldq, sx, Wp, ldp, sa, zp, N, bias, flags, Y, ldy, zw,
                       static_cast<cudaStream_t>(stream), false, false, false);
    if (st == W4A8_OK) t_last_launches = 2;
    return st;
}

static w4a8_status check_g(int M, int K, int N, const uint8_t *Wp, int ldp, const float *sa, const int32_t *zp,
                           const float *bias, unsigned flags, const void *Y, int ldy) {
    w4a8_status st = check_common(M, K, N, Wp, ldp, sa, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (!zp || !aligned4(zp)) return W4A8_ERR_INVALID_ARG;
    // the output is a float sum over groups: there is no single INT32 accumulator
    if ((flags & W4A8_OUT_MASK) == W4A8_OUT_S32) return W4A8_ERR_INVALID_ARG;
    return W4A8_OK;
}

w4a8_status w4g_linear(const float *X, int M, int K, int ldx, const uint8_t *Wp, int ldp, const float *sa,
                       const int32_t *zp, int N, const float *bias, unsigned flags, void *Y, int ldy,
                       void *workspace, size_t workspace_bytes, void *stream) {
    w4a8_status st = check_g(M, K, N, Wp, ldp, sa, zp, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldx < K) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!X || !aligned4(X)) return W4A8_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    if (workspace_bytes < w4a8_workspace_size(M, K)) return W4A8_ERR_WORKSPACE;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    const Workspace ws = carve_workspace(workspace, M, K);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the tensor-core form reads the k-permuted INT8 layout
    const bool perm = path_g(M, flags) == W4A8_PATH_TC;
    st = launch_act_quant(X, M, K, ldx, ws.xq, ws.ldq, ws.sx, s, perm);
    if (st != W4A8_OK) return st;
    st = run_product_g(ws.xq, M, K, ws.ldq, ws.sx, Wp, ldp, sa, zp, N, bias, flags, Y, ldy, s, true, perm);
    if (st == W4A8_OK) t_last_launches = 2;
    return st;
}

w4a8_status w4g_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx, const uint8_t *Wp, int ldp,
                         const float *sa, const int32_t *zp, int N, const float *bias, unsigned flags, void *Y,
                         int ldy, void *stream) {
    w4a8_status st = check_g(M, K, N, Wp, ldp, sa, zp, bias, flags, Y, ldy);
    if (st != W4A8_OK) return st;
    if (ldq < K || ldq % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (M == 0) { t_last_launches = 0; t_last_kernel = ""; return W4A8_OK; }
    if (!Xq || !sx || !aligned16(Xq) || !aligned4(sx)) return W4A8_ERR_INVALID_ARG;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    return run_product_g(Xq, M, K, ldq, sx, Wp, ldp, sa, zp, N, bias, flags, Y, ldy,
                         static_cast<cudaStream_t>(stream), false);
}

unsigned w4a8_last_path(void) { return t_last_path; }

unsigned w4a8_last_launch_count(void) { return t_last_launches; }

const char *w4a8_last_kernel(void) { return t_last_kernel; }

w4a8_status w4a8_linear_grouped(const w4a8_problem *probs, int count, unsigned flags, void *stream) {
    if (count < 0 || (count > 0 && !probs)) return W4A8_ERR_INVALID_ARG;
    if (flags & W4A8_PATH_MASK) return W4A8_ERR_INVALID_ARG;
    bool any = false;
    // every problem is checked before anything is enqueued
    for (int i = 0; i < count; ++i) {
        const w4a8_problem &p = probs[i];
        w4a8_status st = check_common(p.M, p.K, p.N, p.Wp, p.ldp, p.sw, p.bias, flags, p.Y, p.ldy);
        if (st != W4A8_OK) return st;
        if (p.M > 4 || p.ldx < p.K) return W4A8_ERR_INVALID_ARG;
        if (p.M == 0) continue;
        any = true;
        if (!p.X || !aligned4(p.X)) return W4A8_ERR_INVALID_ARG;
        if (p.K > dbulk::X16_MAX_K) return W4A8_ERR_UNSUPPORTED;
        if ((long long)fq_rows(p.M) * dbulk::Geometry(p.K).pitch + dbulk::GROUPED_SLOT > dbulk::SMEM_BUDGET)
            return W4A8_ERR_UNSUPPORTED;
    }
    if (!any) {  // nothing to do
        t_last_launches = 0;
        t_last_kernel = "";
        return W4A8_OK;
    }
    if (!device_info().ok || tc::encode_fn() == nullptr) return W4A8_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned launches = 0;
    w4a8_problem chunk[dbulk::MAX_GROUPED];
    int n = 0;
    for (int i = 0; i <= count; ++i) {
        if (i < count && probs[i].M > 0) chunk[n++] = probs[i];
        if (n == dbulk::MAX_GROUPED || (i == count && n > 0)) {
            w4a8_status st = launch_grouped_chunk(chunk, n, flags, s);
            if (st != W4A8_OK) return st;
            ++launches;
            n = 0;
        }
    }
    t_last_path = W4A8_PATH_DECODE;
    t_last_launches = launches;
    t_last_kernel = "k_decode_grouped";
    return W4A8_OK;
}

w4a8_status w4a8_selftest_timeout(long long cycles, void *stream) {
    if (cycles < 1000 || cycles > ptx::WAIT_LIMIT_CYCLES) return W4A8_ERR_INVALID_ARG;
    if (!device_info().ok) return W4A8_ERR_UNSUPPORTED;
    k_selftest_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cycles);
    return from_cuda(cudaGetLastError());
}

w4a8_status w4a8_get_device_status(int clear, void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return W4A8_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return W4A8_ERR_CUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return W4A8_ERR_CUDA;
    }
    return v;
}

const char *w4a8_status_string(w4a8_status s) {
    switch (s) {
        case W4A8_OK: return "ok";
        case W4A8_ERR_INVALID_ARG: return "invalid argument";
        case W4A8_ERR_UNSUPPORTED: return "unsupported device or shape";
        case W4A8_ERR_WORKSPACE: return "workspace missing or too small";
        case W4A8_ERR_CUDA: return "CUDA error";
        case W4A8_ERR_TIMEOUT: return "bounded wait in a kernel ran out";
        default: return "unknown status";
    }
}

}  // extern "C"
