// gdla_prologue.cu - the projections that make the attention's inputs from the
// hidden state (the fused prologue), for sm_100a.
//
// Method (aitrends.kr/articles/94908, GDLA query-path paragraph: c^Q =
// RMSNorm(x W^Q_a), expanded to content and rotary queries; [c^KV; k^R] = x W^KV_a,
// c^KV RMSNorm'd once and expanded to the KV heads, k^R shared by every head;
// head-configuration paragraph: hidden 4096, query / KV low-rank 1024 / 512, rotary
// 64 of the 192 query-key dims; group-ratio paragraph: lambda = sigmoid(x W^lambda)).
// Readings: RMSNorm eps 1e-6 with a learned weight; rotary embedding in the
// rotate-half form (pair i, i+32) with base 10000, positions from 0 in each
// sequence; gate logits = x W^G; query heads ordered signal 0..4H-1, noise 0..H-1.
//
// Launches (all weights [out_features, in_features] bf16, K-major):
//   1-4  projections of x (K = 4096): c^Q and [c^KV; k^R] (fp32, to the workspace),
//        lambda (sigmoid, fp32 [N, 4H]) and the gate logits (bf16 [N, 4H, 128]);
//   5    per token: RMSNorm of c^Q and c^KV (bf16, with their weights), the rotary
//        angle table cos/sin(t base^(-i/32)) (angles in fp64) and the rotated k^R;
//   6    RMSNorm(c^Q) W^Q_b (K = 1024), one 192-column query head per tile, its
//        rotary 64 columns rotated in the epilogue -> q_sig [N, 4H, 192], q_noise [N, H, 192];
//   7    RMSNorm(c^KV) [W^UK_j; W^UV_j] (K = 512), one KV head per 256-column tile ->
//        k [N, H, 192] = [k_nope | rotated k^R], v [N, H, 128].
// The GEMM: one CTA per 128-row x NT-column tile; a TMA producer warp streams
// 64-wide K chunks of A (the rows) and B (the weights' rows) through a 4-stage
// ring; one elected thread issues tcgen05 MMAs (M = 128, N = NT, fp32 in TMEM);
// the 4 epilogue warps (one TMEM lane = one row) apply the mode's epilogue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

// Epilogue modes of the projection GEMM.
enum : int { PRO_PLAIN = 0, PRO_LAMBDA = 1, PRO_GATE = 2, PRO_QUP = 3, PRO_KVUP = 4 };

// 32 fp32 values (as bits) -> 32 bf16 at dst (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_bf16_32(__nv_bfloat16 *dst, const uint32_t (&o)[32]) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        d4[i] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * i]), __uint_as_float(o[8 * i + 1])),
                           pack_bf16x2(__uint_as_float(o[8 * i + 2]), __uint_as_float(o[8 * i + 3])),
                           pack_bf16x2(__uint_as_float(o[8 * i + 4]), __uint_as_float(o[8 * i + 5])),
                           pack_bf16x2(__uint_as_float(o[8 * i + 6]), __uint_as_float(o[8 * i + 7])));
}

namespace pg {
constexpr int STAGES = 4;
constexpr int A_CHUNK = 128 * 128;  // 128 rows x 64 K (bf16)
constexpr int NUM_THREADS = 192;    // epilogue warps 0-3, producer 4, MMA 5
constexpr int PRODUCER_WARP = 4, MMA_WARP = 5;
constexpr int ROPE_HALF = 32;
}  // namespace pg

template <int EPI, int NT>
struct ProjCfg {
    static constexpr int B_CHUNK = NT * 128;
    static constexpr int STAGE = pg::A_CHUNK + B_CHUNK;
    static constexpr int OFF_BAR = pg::STAGES * STAGE;
    static constexpr int OFF_MISC = OFF_BAR + 16 * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
    static constexpr uint32_t TMEM_COLS = NT <= 32 ? 32 : (NT <= 64 ? 64 : (NT <= 128 ? 128 : 256));
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(NT % 32 == 0 && NT <= 256, "tile width");
};

// Position of packed row m in its sequence (starts[] = cumulative sequence starts).
__device__ __forceinline__ int row_position(const ProloguePlan &p, int m) {
    int lo = 0, hi = p.n_seqs;  // starts[lo] <= m < starts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.starts[mid] <= m) lo = mid; else hi = mid;
    }
    return m - p.starts[lo];
}

template <int EPI, int NT>
__global__ void __launch_bounds__(pg::NUM_THREADS, 1)
gdla_proj_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_b2, const PrologueIO io, int M, int K) {
    using C = ProjCfg<EPI, NT>;
    using namespace pg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars;               // [stage]
    uint64_t *empty = bars + STAGES;     // [stage]
    uint64_t *mma_done = bars + 2 * STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * 128, tile_n = blockIdx.y, n0 = tile_n * NT;
    const int nk = K / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            int issued = 0;
            for (int kc = 0; kc < nk; ++kc) {
                const int st = kc % STAGES;
                if (kc >= STAGES && !mbar_wait(empty + st, ((kc / STAGES) + 1) & 1, abort_flag, ERR_SITE_PROLOGUE | 1))
                    break;
                mbar_arrive_expect_tx(full + st, C::STAGE);
                uint8_t *sb = smem + st * C::STAGE;
                tma_load_3d(sb, &tm_a, full + st, kc * 64, m0, 0);
                if (EPI == PRO_KVUP) {  // [W^UK_j; W^UV_j]: two 128-row boxes
                    tma_load_3d(sb + A_CHUNK, &tm_b, full + st, kc * 64, tile_n * 128, 0);
                    tma_load_3d(sb + A_CHUNK + 128 * 128, &tm_b2, full + st, kc * 64, tile_n * 128, 0);
                } else {
                    tma_load_3d(sb + A_CHUNK, &tm_b, full + st, kc * 64, n0, 0);
                }
                issued = kc + 1;
            }
            if (*abort_flag)
                for (int k = max(0, issued - STAGES); k < issued; ++k)
                    mbar_wait_cycles(full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
        }
    } else if (warp == MMA_WARP) {
        const uint32_t leader = elect_one_sync();
        constexpr uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
        const uint64_t a_desc0 = desc_sw128(smem_u32(smem), 16, 1024);
        const uint64_t b_desc0 = desc_sw128(smem_u32(smem + A_CHUNK), 16, 1024);
        bool ok = true;
        for (int kc = 0; kc < nk; ++kc) {
            const int st = kc % STAGES;
            if (!__all_sync(0xffffffffu, mbar_wait(full + st, (kc / STAGES) & 1, abort_flag, ERR_SITE_PROLOGUE | 2))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sb = st * C::STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_ss_leader(tmem, a_desc0 + ((sb + kk * 32) >> 4), b_desc0 + ((sb + kk * 32) >> 4), idesc,
                               (kc > 0 || kk > 0) ? 1u : 0u, leader);
            umma_commit_leader(empty + st, leader);
        }
        if (ok) umma_commit_leader(mma_done, leader);
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int m = m0 + warp * 32 + lane;
        const bool row_ok = m < M;
        if (__all_sync(0xffffffffu, mbar_wait(mma_done, 0, abort_flag, ERR_SITE_PROLOGUE | 3))) {
            tc_fence_after();
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            if constexpr (EPI == PRO_PLAIN) {
                float *dst = io.f32_out + static_cast<size_t>(m) * io.ld_out + n0;
#pragma unroll 1
                for (int ch = 0; ch < NT / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + ch * 32, o);
                    if (row_ok) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + ch * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            d4[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
                    }
                }
            } else if constexpr (EPI == PRO_LAMBDA) {
#pragma unroll 1
                for (int ch = 0; ch < NT / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + ch * 32, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = n0 + ch * 32 + i;
                        if (row_ok && n < io.n_out)
                            io.lambda[static_cast<size_t>(m) * io.n_out + n] =
                                1.f / (1.f + __expf(-__uint_as_float(o[i])));
                    }
                }
            } else if constexpr (EPI == PRO_GATE) {
                __nv_bfloat16 *dst = io.gate + static_cast<size_t>(m) * io.n_out + n0;
#pragma unroll 1
                for (int ch = 0; ch < NT / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + ch * 32, o);
                    if (row_ok) {
                        uint4 *d4 = reinterpret_cast<uint4 *>(dst + ch * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            d4[i] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * i]), __uint_as_float(o[8 * i + 1])),
                                               pack_bf16x2(__uint_as_float(o[8 * i + 2]), __uint_as_float(o[8 * i + 3])),
                                               pack_bf16x2(__uint_as_float(o[8 * i + 4]), __uint_as_float(o[8 * i + 5])),
                                               pack_bf16x2(__uint_as_float(o[8 * i + 6]), __uint_as_float(o[8 * i + 7])));
                    }
                }
            } else if constexpr (EPI == PRO_QUP) {
                // one query head: content dims 0..127, rotary dims 128..191 (pairs i, i+32)
                const int h = tile_n;
                __nv_bfloat16 *dst = (h < 4 * io.hkv)
                                         ? io.q_sig + (static_cast<size_t>(m) * 4 * io.hkv + h) * 192
                                         : io.q_noise + (static_cast<size_t>(m) * io.hkv + (h - 4 * io.hkv)) * 192;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + ch * 32, o);
                    if (row_ok) store_bf16_32(dst + ch * 32, o);
                }
                uint32_t a[32], b[32];
                tmem_ld32(lane_base + 128, a);
                tmem_ld32(lane_base + 160, b);
                if (row_ok) {
                    const float *rot = io.rot + static_cast<size_t>(m) * 64;  // cos 0..31, sin 32..63
                    uint32_t ra[32], rb[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float c = __ldg(rot + i), s = __ldg(rot + 32 + i);
                        const float x0 = __uint_as_float(a[i]), x1 = __uint_as_float(b[i]);
                        ra[i] = __float_as_uint(x0 * c - x1 * s);
                        rb[i] = __float_as_uint(x0 * s + x1 * c);
                    }
                    store_bf16_32(dst + 128, ra);
                    store_bf16_32(dst + 160, rb);
                }
            } else {  // PRO_KVUP: one KV head j: k_nope (cols 0..127), v (128..255), rotated k^R copied
                const int j = tile_n;
                __nv_bfloat16 *kd = io.k + (static_cast<size_t>(m) * io.hkv + j) * 192;
                __nv_bfloat16 *vd = io.v + (static_cast<size_t>(m) * io.hkv + j) * 128;
#pragma unroll 1
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + ch * 32, o);
                    if (row_ok) store_bf16_32(ch < 4 ? kd + ch * 32 : vd + (ch - 4) * 32, o);
                }
                if (row_ok) {
                    const uint4 *kr = reinterpret_cast<const uint4 *>(io.krope + static_cast<size_t>(m) * 64);
                    uint4 *kdst = reinterpret_cast<uint4 *>(kd + 128);
#pragma unroll
                    for (int i = 0; i < 8; ++i) kdst[i] = __ldg(kr + i);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Per token (one warp): RMSNorm of c^Q (1024) and c^KV (512) with their weights
// into bf16 rows, the rotary table cos/sin(t base^(-i/32)) for i < 32 (angles and
// their sine / cosine in fp64, stored fp32), and k^R rotated (bf16).
__global__ void __launch_bounds__(256)
gdla_prologue_norm_kernel(const PrologueIO io, const ProloguePlan plan, int M) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= M) return;
    const int m = warp;
    const float *cq = io.cq + static_cast<size_t>(m) * 1024;
    const float *ckv = io.ckv + static_cast<size_t>(m) * 576;
    float ss = 0.f;
    for (int i = lane; i < 1024; i += 32) ss = fmaf(cq[i], cq[i], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rq = rsqrtf(ss * (1.f / 1024.f) + 1e-6f);
    for (int i = lane; i < 1024; i += 32)
        io.cq_n[static_cast<size_t>(m) * 1024 + i] = __float2bfloat16_rn(cq[i] * rq * io.gamma_q[i]);
    ss = 0.f;
    for (int i = lane; i < 512; i += 32) ss = fmaf(ckv[i], ckv[i], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rkv = rsqrtf(ss * (1.f / 512.f) + 1e-6f);
    for (int i = lane; i < 512; i += 32)
        io.ckv_n[static_cast<size_t>(m) * 512 + i] = __float2bfloat16_rn(ckv[i] * rkv * io.gamma_kv[i]);
    // rotary table and k^R (lane = pair i of 32)
    const double inv = exp2(-static_cast<double>(lane) * (13.287712379549449 / 32.0));  // 10000^(-i/32)
    double s, c;
    sincos(static_cast<double>(row_position(plan, m)) * inv, &s, &c);
    io.rot[static_cast<size_t>(m) * 64 + lane] = static_cast<float>(c);
    io.rot[static_cast<size_t>(m) * 64 + 32 + lane] = static_cast<float>(s);
    const float x0 = ckv[512 + lane], x1 = ckv[512 + 32 + lane];
    io.krope[static_cast<size_t>(m) * 64 + lane] =
        __float2bfloat16_rn(static_cast<float>(x0 * c - x1 * s));
    io.krope[static_cast<size_t>(m) * 64 + 32 + lane] =
        __float2bfloat16_rn(static_cast<float>(x0 * s + x1 * c));
}

// ------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------
template <int EPI, int NT>
static cudaError_t launch_proj(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &b2,
                               const PrologueIO &io, int M, int K, int n_tiles, cudaStream_t stream) {
    using C = ProjCfg<EPI, NT>;
    static PerContextFlag attr_set;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        e = cudaFuncSetAttribute(gdla_proj_kernel<EPI, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    dim3 grid((M + 127) / 128, n_tiles);
    gdla_proj_kernel<EPI, NT><<<grid, pg::NUM_THREADS, C::SMEM_BYTES, stream>>>(a, b, b2, io, M, K);
    return cudaPeekAtLastError();
}

cudaError_t launch_prologue(const PrologueLaunch &L, const ProloguePlan &plan, int M, cudaStream_t stream) {
    PrologueIO io = L.io;
    const int hkv = io.hkv;
    cudaError_t e;
    // 1-4: projections of x
    io.f32_out = io.cq, io.ld_out = 1024;
    if ((e = launch_proj<PRO_PLAIN, 256>(L.tm_x, L.tm_wqa, L.tm_wqa, io, M, 4096, 4, stream)) != cudaSuccess) return e;
    io.f32_out = io.ckv, io.ld_out = 576;
    if ((e = launch_proj<PRO_PLAIN, 192>(L.tm_x, L.tm_wkva, L.tm_wkva, io, M, 4096, 3, stream)) != cudaSuccess) return e;
    io.n_out = 4 * hkv;
    if ((e = launch_proj<PRO_LAMBDA, 64>(L.tm_x, L.tm_wlam, L.tm_wlam, io, M, 4096, (4 * hkv + 63) / 64, stream)) !=
        cudaSuccess)
        return e;
    io.n_out = 4 * hkv * 128;
    if ((e = launch_proj<PRO_GATE, 256>(L.tm_x, L.tm_wgate, L.tm_wgate, io, M, 4096, 2 * hkv, stream)) != cudaSuccess)
        return e;
    // 5: norms, rotary table, rotated k^R
    gdla_prologue_norm_kernel<<<(M + 7) / 8, 256, 0, stream>>>(io, plan, M);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    // 6-7: up-projections
    if ((e = launch_proj<PRO_QUP, 192>(L.tm_cqn, L.tm_wqb, L.tm_wqb, io, M, 1024, 5 * hkv, stream)) != cudaSuccess)
        return e;
    return launch_proj<PRO_KVUP, 256>(L.tm_ckvn, L.tm_wuk, L.tm_wuv, io, M, 512, hkv, stream);
}

}  // namespace gdla
