// gdla_decode.cu - varlen split-KV GDLA decode for sm_100a.
//
// One query token per sequence (position L_b - 1, the cache holding it). For
// each (sequence b, KV group j, split s) a CTA streams its slice of K_j/V_j
// through shared memory (TMA, 64 keys per stage) and computes, for the five
// query heads of the group at once, the split's running max m, sum l and
// unnormalised O. The dense contractions run on tensor cores with the keys as
// the MMA's M dimension:
//     S^T[16 keys x 8 heads]  = K[16 x 192] . Q^T[192 x 8]      (5 of 8 columns live)
//     O^T[128 dv x 8 heads]  += V^T[128 x 16 keys] . P^T[16 x 8]
// P^T is transposed in registers (movmatrix) into the B fragment of the PV
// product. A second, small kernel merges the splits with a warp-shuffle
// log-sum-exp reduction and applies the GDLA epilogue (D = H_S - lambda H_N,
// sigmoid gate, bf16). When one split covers every key (sliding window, short
// caches) the split kernel applies the epilogue itself.
//
// Method: aitrends.kr/articles/94908, GDLA paragraphs (shared KV head per
// group, D_t = H_S,t - lambda_t Repeat_g(H_N,t), query-based gate).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

namespace dc {
constexpr int DQK = 192, DV = 128, HEADS = 5;
constexpr int TK = 64;                     // keys per stage
constexpr int STAGES = 2;
constexpr int CONSUMER_WARPS = 4;          // each takes 16 keys of a stage
constexpr int NUM_THREADS = (CONSUMER_WARPS + 1) * 32;
constexpr int K_CHUNK = TK * 128;          // one 64-dim swizzled chunk: 8 KB
constexpr int K_STAGE = 3 * K_CHUNK;       // 24 KB
constexpr int V_STAGE = 2 * K_CHUNK;       // 16 KB
constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + STAGES * K_STAGE;
constexpr int OFF_RED = OFF_V + STAGES * V_STAGE;                 // [4 warps][5 heads][128] fp32
constexpr int RED_BYTES = CONSUMER_WARPS * HEADS * DV * 4;
constexpr int OFF_ML = OFF_RED + RED_BYTES;                        // [4 warps][8 heads] m, l
constexpr int OFF_BAR = OFF_ML + 2 * CONSUMER_WARPS * 8 * 4;
constexpr int OFF_MISC = OFF_BAR + 2 * STAGES * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr uint32_t STAGE_TX = K_STAGE + V_STAGE;
}  // namespace dc

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of (row, 16-byte unit) inside a 128-byte-swizzled [rows x 128 B] chunk.
__device__ __forceinline__ uint32_t swz(int row, int unit) {
    return static_cast<uint32_t>(row * 128 + ((unit ^ (row & 7)) << 4));
}

// GDLA epilogue for one sequence/group, given the 5 normalised heads in smem
// (h[5][128]: signal 0..3, noise 4). 128 threads, one per dv element.
__device__ __forceinline__ void decode_epilogue(const float *h, const float *__restrict__ lambda,
                                                const __nv_bfloat16 *__restrict__ gate,
                                                __nv_bfloat16 *__restrict__ out, size_t row0, int d) {
    const float hn = h[4 * dc::DV + d];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const size_t row = row0 + i;
        const float lam = lambda[row];
        const float g = __bfloat162float(gate[row * dc::DV + d]);
        const float dd = h[i * dc::DV + d] - lam * hn;
        out[row * dc::DV + d] = __float2bfloat16_rn(__fdividef(dd, 1.f + __expf(-g)));
    }
}

__global__ void __launch_bounds__(dc::NUM_THREADS, 2)
gdla_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __nv_bfloat16 *__restrict__ q_sig, const __nv_bfloat16 *__restrict__ q_noise,
                         const int32_t *__restrict__ cu_seqlens_k, const float *__restrict__ lambda,
                         const __nv_bfloat16 *__restrict__ gate, __nv_bfloat16 *__restrict__ out,
                         float *__restrict__ ws, const DecodePlan plan) {
    using namespace dc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *empty = full + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC);
    float *red = reinterpret_cast<float *>(smem + OFF_RED);
    float *ml = reinterpret_cast<float *>(smem + OFF_ML);

    const int split = blockIdx.x;
    const int group = blockIdx.y;
    const int b = blockIdx.z;
    const int hkv = plan.hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int start = cu_seqlens_k[b];
    const int len = cu_seqlens_k[b + 1] - start;
    const bool len_ok = (start >= 0) && (len >= 1) && (len <= plan.max_seqlen_k) &&
                        (cu_seqlens_k[b + 1] <= plan.num_cache_rows);
    const int lo = (plan.window > 0) ? max(0, len - plan.window) : 0;
    const int k_begin = lo + split * plan.split_keys;
    const int k_end = len_ok ? min(len, k_begin + plan.split_keys) : k_begin;
    const int n_keys = max(0, k_end - k_begin);
    const int n_stages = (n_keys + TK - 1) / TK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, CONSUMER_WARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CONSUMER_WARPS) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0 && n_stages > 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued = 0;
            for (int it = 0; it < n_stages; ++it) {
                const int st = it % STAGES;
                if (it >= STAGES &&
                    !mbar_wait(empty + st, ((it / STAGES) + 1) & 1, abort_flag, ERR_SITE_DECODE | 1))
                    break;
                mbar_arrive_expect_tx(full + st, STAGE_TX);
                const int row = start + k_begin + it * TK;
                for (int c = 0; c < 3; ++c)
                    tma_load_3d(smem + OFF_K + st * K_STAGE + c * K_CHUNK, &tm_k, full + st, c * 64, group, row);
                for (int c = 0; c < 2; ++c)
                    tma_load_3d(smem + OFF_V + st * V_STAGE + c * K_CHUNK, &tm_v, full + st, c * 64, group, row);
                issued = it + 1;
            }
            if (*abort_flag)
                for (int it = max(0, issued - STAGES); it < issued; ++it)
                    mbar_wait_cycles(full + it % STAGES, (it / STAGES) & 1, 1ll << 22);
        }
    } else {
        // ------------------------------- consumers --------------------------------
        const int g = lane >> 2, c = lane & 3;
        // Q^T fragments (B operand): thread holds head g, dims 16*ks + 2c(+1) and +8.
        uint32_t qf[DQK / 16][2];
        {
            const __nv_bfloat16 *qrow = nullptr;
            if (g < 4) qrow = q_sig + (static_cast<size_t>(b) * 4 * hkv + 4 * group + g) * DQK;
            else if (g == 4) qrow = q_noise + (static_cast<size_t>(b) * hkv + group) * DQK;
#pragma unroll
            for (int ks = 0; ks < DQK / 16; ++ks) {
                if (qrow) {
                    qf[ks][0] = *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + 2 * c);
                    qf[ks][1] = *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + 8 + 2 * c);
                } else {
                    qf[ks][0] = 0u;
                    qf[ks][1] = 0u;
                }
            }
        }
        const float c_log2 = 0.07216878364870322f * 1.4426950408889634f;  // log2(e) / sqrt(192)
        float o[DV / 16][4];
#pragma unroll
        for (int mt = 0; mt < DV / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of heads 2c, 2c+1
        float l0 = 0.f, l1 = 0.f;              // this thread's partial sums

        const int mi = lane >> 3, ri = lane & 7;
        for (int it = 0; it < n_stages; ++it) {
            const int st = it % STAGES;
            if (!mbar_wait(full + st, (it / STAGES) & 1, abort_flag, ERR_SITE_DECODE | 2)) break;
            const uint32_t kb = smem_u32(smem + OFF_K + st * K_STAGE);
            const uint32_t vb = smem_u32(smem + OFF_V + st * V_STAGE);
            const int key0 = warp * 16;  // this warp's 16 keys within the stage
            // S^T = K Q^T
            float s[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int krow = key0 + ri + 8 * (mi & 1);
#pragma unroll
                for (int ks = 0; ks < DQK / 16; ++ks) {
                    const int dim = ks * 16 + 8 * (mi >> 1);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(kb + (dim >> 6) * K_CHUNK + swz(krow, (dim & 63) >> 3), a0, a1, a2, a3);
                    mma_bf16(s, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                }
            }
            // mask keys past the split end (and the cache rows of other sequences)
            const int ubase = k_begin + it * TK + key0;
            if (ubase + g >= k_end) { s[0] = -INFINITY; s[1] = -INFINITY; }
            if (ubase + g + 8 >= k_end) { s[2] = -INFINITY; s[3] = -INFINITY; }
            float mx0 = fmaxf(s[0], s[2]) * c_log2, mx1 = fmaxf(s[1], s[3]) * c_log2;
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
            const float a0s = (n0 == -INFINITY) ? 1.f : fast_exp2(m0 - n0);
            const float a1s = (n1 == -INFINITY) ? 1.f : fast_exp2(m1 - n1);
            m0 = n0;
            m1 = n1;
            const float b0 = (n0 == -INFINITY) ? 0.f : n0, b1 = (n1 == -INFINITY) ? 0.f : n1;
            const float p0 = fast_exp2(fmaf(s[0], c_log2, -b0));
            const float p1 = fast_exp2(fmaf(s[1], c_log2, -b1));
            const float p2 = fast_exp2(fmaf(s[2], c_log2, -b0));
            const float p3 = fast_exp2(fmaf(s[3], c_log2, -b1));
            l0 = l0 * a0s + p0 + p2;
            l1 = l1 * a1s + p1 + p3;
#pragma unroll
            for (int mt = 0; mt < DV / 16; ++mt) {
                o[mt][0] *= a0s;
                o[mt][1] *= a1s;
                o[mt][2] *= a0s;
                o[mt][3] *= a1s;
            }
            // P^T blocks (keys g / g+8, heads 2c..2c+1) -> transposed B fragments
            const uint32_t pb0 = movmatrix_t(pack_bf16x2(p0, p1));
            const uint32_t pb1 = movmatrix_t(pack_bf16x2(p2, p3));
            {
                const int vrow = key0 + ri + 8 * (mi >> 1);
#pragma unroll
                for (int mt = 0; mt < DV / 16; ++mt) {
                    const int dv = mt * 16 + 8 * (mi & 1);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(vb + (dv >> 6) * K_CHUNK + swz(vrow, (dv & 63) >> 3), a0, a1, a2, a3);
                    mma_bf16(o[mt], a0, a1, a2, a3, pb0, pb1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + st);
        }
        // ---- merge the four warps: per head max, then rescaled sums ----
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
        if (g == 0) {
            ml[(warp * 8 + 2 * c) * 2 + 0] = m0;
            ml[(warp * 8 + 2 * c) * 2 + 1] = l0;
            ml[(warp * 8 + 2 * c + 1) * 2 + 0] = m1;
            ml[(warp * 8 + 2 * c + 1) * 2 + 1] = l1;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // global max over warps for this thread's two heads
        float gm0 = -INFINITY, gm1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < CONSUMER_WARPS; ++w) {
            gm0 = fmaxf(gm0, ml[(w * 8 + 2 * c) * 2]);
            gm1 = fmaxf(gm1, ml[(w * 8 + 2 * c + 1) * 2]);
        }
        const float f0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - gm0);
        const float f1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - gm1);
        // write this warp's rescaled O^T (heads < 5) to red[warp][head][dv]
        float *rw = red + warp * HEADS * DV;
#pragma unroll
        for (int mt = 0; mt < DV / 16; ++mt) {
            const int dv0 = mt * 16 + g;
            if (2 * c < HEADS) {
                rw[(2 * c) * DV + dv0] = o[mt][0] * f0;
                rw[(2 * c) * DV + dv0 + 8] = o[mt][2] * f0;
            }
            if (2 * c + 1 < HEADS) {
                rw[(2 * c + 1) * DV + dv0] = o[mt][1] * f1;
                rw[(2 * c + 1) * DV + dv0 + 8] = o[mt][3] * f1;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // thread d (0..127) sums the 4 warps for every head, fixed order
        const int d = threadIdx.x;
        float hsum[HEADS];
        float hm[HEADS], hl[HEADS];
#pragma unroll
        for (int h = 0; h < HEADS; ++h) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < CONSUMER_WARPS; ++w) M = fmaxf(M, ml[(w * 8 + h) * 2]);
            float Ls = 0.f, Os = 0.f;
#pragma unroll
            for (int w = 0; w < CONSUMER_WARPS; ++w) {
                const float mw = ml[(w * 8 + h) * 2];
                const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
                Ls += ml[(w * 8 + h) * 2 + 1] * f;
                Os += red[(w * HEADS + h) * DV + d];
            }
            hm[h] = M;
            hl[h] = Ls;
            hsum[h] = Os;
        }
        const size_t slot = (static_cast<size_t>(b) * hkv + group) * plan.num_splits + split;
        if (plan.num_splits == 1) {
            // one split holds every key: finish here. Reuse red[0] as h[5][128].
            asm volatile("bar.sync 1, 128;" ::: "memory");
            float *hbuf = red;
#pragma unroll
            for (int h = 0; h < HEADS; ++h) hbuf[h * DV + d] = (hl[h] > 0.f) ? hsum[h] / hl[h] : 0.f;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            decode_epilogue(hbuf, lambda, gate, out, (static_cast<size_t>(b) * hkv + group) * 4, d);
        } else {
            float *wo = ws + slot * (HEADS * DV);
            float *wml = ws + plan.ml_offset_floats + slot * (HEADS * 2);
#pragma unroll
            for (int h = 0; h < HEADS; ++h) wo[h * DV + d] = hsum[h];
            if (d < HEADS) {
                wml[d * 2 + 0] = hm[d];
                wml[d * 2 + 1] = hl[d];
            }
        }
    }
}

// Split merge: one CTA of 5 warps per (sequence, group); warp h merges head h.
// Lanes walk the splits (32 at a time): a shuffle max gives the global m, each
// split gets weight exp2(m_s - m), and each lane then owns 4 dv columns of the
// weighted sum. Splits that saw no key carry m = -inf and are skipped.
__global__ void __launch_bounds__(160)
gdla_decode_combine_kernel(const float *__restrict__ ws, const float *__restrict__ lambda,
                           const __nv_bfloat16 *__restrict__ gate, __nv_bfloat16 *__restrict__ out,
                           const DecodePlan plan) {
    using namespace dc;
    __shared__ float hbuf[HEADS * DV];
    __shared__ float wsh[HEADS][64];
    const int group = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hkv = plan.hkv;
    const int ns = plan.num_splits;
    const size_t slot0 = (static_cast<size_t>(b) * hkv + group) * ns;
    const float *wml = ws + plan.ml_offset_floats;
    const int h = warp;
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, wml[(slot0 + s) * (HEADS * 2) + h * 2]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float Lsum = 0.f;
    for (int s = lane; s < ns; s += 32) {
        const float ms = wml[(slot0 + s) * (HEADS * 2) + h * 2];
        const float ls = wml[(slot0 + s) * (HEADS * 2) + h * 2 + 1];
        const float w = (ms == -INFINITY) ? 0.f : fast_exp2(ms - M);
        wsh[h][s] = w;
        Lsum += ls * w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
    __syncwarp();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < ns; ++s) {
        const float w = wsh[h][s];
        if (w == 0.f) continue;
        const float4 v = *reinterpret_cast<const float4 *>(ws + (slot0 + s) * (HEADS * DV) + h * DV + lane * 4);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
    }
    const float inv = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) hbuf[h * DV + lane * 4 + i] = acc[i] * inv;
    __syncthreads();
    if (threadIdx.x < DV) decode_epilogue(hbuf, lambda, gate, out, (static_cast<size_t>(b) * hkv + group) * 4,
                                          threadIdx.x);
}

int decode_smem_bytes() { return dc::SMEM_BYTES; }

cudaError_t launch_decode(const DecodeLaunch &L, const DecodePlan &plan, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(gdla_decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.num_splits, plan.hkv, plan.batch);
    gdla_decode_split_kernel<<<grid, dc::NUM_THREADS, dc::SMEM_BYTES, stream>>>(
        L.tm_k, L.tm_v, L.q_sig, L.q_noise, L.cu_seqlens_k, L.lambda, L.gate, L.out, L.ws, plan);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess || plan.num_splits == 1) return e;
    dim3 grid2(plan.hkv, plan.batch);
    gdla_decode_combine_kernel<<<grid2, 160, 0, stream>>>(L.ws, L.lambda, L.gate, L.out, plan);
    return cudaPeekAtLastError();
}

}  // namespace gdla
