// gdla_prefill.cu - packed varlen GDLA prefill for sm_100a.
//
// Method (aitrends.kr/articles/94908, GDLA paragraphs): for each KV head j the
// 4 signal heads 4j..4j+3 and the noise head j run causal softmax attention
// over the same K_j (192) and V_j (128); then D_i = H_S,i - lambda_i * H_N,j
// and out_i = sigmoid(gate_i) * D_i.
//
// Tiling. One CTA owns one KV group and a tile of TOK = 24 consecutive tokens
// of one sequence. The 5 query heads of those tokens are packed into the M =
// 128 rows of one tensor-core tile:
//     rows 0..95    signal heads, row = 4*tau + h   (tau = token in tile, h = 0..3)
//     rows 96..119  the noise head, row = 96 + tau
//     rows 120..127 unused (zero queries)
// so every K/V tile is staged once into shared memory (TMA) and consumed by
// all five heads, and one tcgen05 MMA covers them all. For each key tile:
//     S = Q K^T        (tcgen05, M=128 N=128 K=192, A and B from smem, D in TMEM)
//     softmax warps    (one TMEM lane = one row; online max/sum, P = exp2 -> bf16 into TMEM)
//     O += P V         (tcgen05, A = P from TMEM, B = V from smem, MN-major)
// The epilogue finalises O / l, exchanges the noise rows through shared
// memory, and writes sigmoid(g) * (H_S - lambda H_N) as bf16.
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue, warp 4 TMA producer,
// warp 5 TMEM allocation + MMA issue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

namespace pf {
constexpr int TOK = kPrefillTileTokens;  // tokens per CTA tile
constexpr int ROWS = 128;                // tensor-core M
constexpr int SIG_ROWS = 4 * TOK;        // 96
constexpr int NOISE_ROW0 = SIG_ROWS;     // 96
constexpr int BN = 128;                  // keys per KV tile
constexpr int DQK = 192, DV = 128;
constexpr int KCHUNKS = DQK / 64;        // 128-byte swizzle chunks of a K row
constexpr int VCHUNKS = DV / 64;

constexpr int Q_CHUNK_BYTES = ROWS * 128;          // 16 KB
constexpr int Q_BYTES = KCHUNKS * Q_CHUNK_BYTES;   // 48 KB
constexpr int K_CHUNK_BYTES = BN * 128;            // 16 KB
constexpr int K_STAGE_BYTES = KCHUNKS * K_CHUNK_BYTES;  // 48 KB
constexpr int V_STAGE_BYTES = VCHUNKS * K_CHUNK_BYTES;  // 32 KB
constexpr int STAGES = 2;

constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_K + STAGES * K_STAGE_BYTES;
constexpr int OFF_BAR = OFF_V + STAGES * V_STAGE_BYTES;
constexpr int NUM_BARS = 15;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack

constexpr int HN_STRIDE = 132;  // floats per noise row in the exchange buffer
static_assert(TOK * HN_STRIDE * 4 <= K_STAGE_BYTES, "noise exchange must fit in a K stage");

constexpr uint32_t Q_TX = KCHUNKS * (64 * 4 * TOK * 2 + 64 * 1 * TOK * 2);
constexpr uint32_t K_TX = K_STAGE_BYTES;
constexpr uint32_t V_TX = V_STAGE_BYTES;

// TMEM columns
constexpr uint32_t O_COL = 0;
constexpr uint32_t S_COL0 = 128;
constexpr uint32_t TMEM_COLS = 512;

constexpr int NUM_THREADS = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
}  // namespace pf

__global__ void __launch_bounds__(pf::NUM_THREADS, 1)
gdla_prefill_kernel(const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_qn,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const float *__restrict__ lambda, const __nv_bfloat16 *__restrict__ gate,
                    __nv_bfloat16 *__restrict__ out, const __grid_constant__ PrefillPlan plan) {
    using namespace pf;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;   // [2]
    uint64_t *k_empty = bars + 3;  // [2]
    uint64_t *v_full = bars + 5;   // [2]
    uint64_t *v_empty = bars + 7;  // [2]
    uint64_t *s_full = bars + 9;   // [2]
    uint64_t *p_full = bars + 11;  // [2]
    uint64_t *o_done = bars + 13;   // one phase per PV product (rescale waits)
    uint64_t *o_final = bars + 14;  // single phase: the last PV product is done (epilogue)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int hkv = plan.hkv;
    const int group = blockIdx.x % hkv;
    const uint32_t item = plan.items[blockIdx.x / hkv];
    const int seq = static_cast<int>(item >> kItemSeqShift);
    const int qt = static_cast<int>(item & kItemTileMask);
    const int s0 = plan.seq_start[seq];
    const int L = plan.seq_len[seq];
    const int t0 = qt * TOK;
    const int window = plan.window;
    const int kv_lo = (window > 0) ? max(0, t0 - window + 1) : 0;
    const int kv_hi = min(L, t0 + TOK);
    const int n_tiles = (kv_hi - kv_lo + BN - 1) / BN;
    const int hs = 4 * hkv;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(k_empty + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(v_empty + i, 1);
            mbar_init(s_full + i, 1);
            mbar_init(p_full + i, 128);
        }
        mbar_init(o_done, 1);
        mbar_init(o_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Rows 120..127 of Q are never loaded: zero them so their (unused) rows stay finite.
    if (warp == 3 && lane >= 24) {
        const int r = 96 + lane;
        for (int c = 0; c < KCHUNKS; ++c) {
            uint4 *dst = reinterpret_cast<uint4 *>(smem + OFF_Q + c * Q_CHUNK_BYTES + r * 128);
            for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_qs);
            tma_prefetch_desc(&tm_qn);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(q_full, Q_TX);
            for (int c = 0; c < KCHUNKS; ++c) {
                uint8_t *qc = smem + OFF_Q + c * Q_CHUNK_BYTES;
                tma_load_3d(qc, &tm_qs, q_full, c * 64, 4 * group, s0 + t0);
                tma_load_3d(qc + NOISE_ROW0 * 128, &tm_qn, q_full, c * 64, group, s0 + t0);
            }
            int issued_k = 0, issued_v = 0;
            for (int k = 0; k < n_tiles; ++k) {
                const int st = k & 1;
                const int row = s0 + kv_lo + k * BN;
                if (k >= 2 && !mbar_wait(k_empty + st, ((k >> 1) + 1) & 1, abort_flag, ERR_SITE_PREFILL | 1)) break;
                mbar_arrive_expect_tx(k_full + st, K_TX);
                for (int c = 0; c < KCHUNKS; ++c)
                    tma_load_3d(smem + OFF_K + st * K_STAGE_BYTES + c * K_CHUNK_BYTES, &tm_k, k_full + st, c * 64,
                                group, row);
                issued_k = k + 1;
                if (k >= 2 && !mbar_wait(v_empty + st, ((k >> 1) + 1) & 1, abort_flag, ERR_SITE_PREFILL | 2)) break;
                mbar_arrive_expect_tx(v_full + st, V_TX);
                for (int c = 0; c < VCHUNKS; ++c)
                    tma_load_3d(smem + OFF_V + st * V_STAGE_BYTES + c * K_CHUNK_BYTES, &tm_v, v_full + st, c * 64,
                                group, row);
                issued_v = k + 1;
            }
            if (*abort_flag) {
                // Another role gave up: let this thread's copies still in flight land
                // before the CTA (and its shared memory) goes away.
                mbar_wait_cycles(q_full, 0, 1ll << 22);
                for (int k = max(0, issued_k - 2); k < issued_k; ++k)
                    mbar_wait_cycles(k_full + (k & 1), (k >> 1) & 1, 1ll << 22);
                for (int k = max(0, issued_v - 2); k < issued_v; ++k)
                    mbar_wait_cycles(v_full + (k & 1), (k >> 1) & 1, 1ll << 22);
            }
        }
    } else if (warp == 5) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(ROWS, BN, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(ROWS, DV, false, true);
            const uint32_t q_base = smem_u32(smem + OFF_Q);
            bool ok = mbar_wait(q_full, 0, abort_flag, ERR_SITE_PREFILL | 3);
            for (int k = 0; ok && k <= n_tiles; ++k) {
                if (k < n_tiles) {
                    const int st = k & 1;
                    if (!mbar_wait(k_full + st, (k >> 1) & 1, abort_flag, ERR_SITE_PREFILL | 4)) break;
                    tc_fence_after();
                    const uint32_t k_base = smem_u32(smem + OFF_K + st * K_STAGE_BYTES);
                    const uint32_t d = tmem + S_COL0 + st * 128;
#pragma unroll
                    for (int kk = 0; kk < DQK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * Q_CHUNK_BYTES + (kk & 3) * 32;
                        const uint32_t offk = (kk >> 2) * K_CHUNK_BYTES + (kk & 3) * 32;
                        umma_ss(d, desc_sw128(q_base + off, 16, 1024), desc_sw128(k_base + offk, 16, 1024), idesc_s,
                                kk > 0);
                    }
                    umma_commit(s_full + st);
                    umma_commit(k_empty + st);
                }
                if (k >= 1) {
                    const int j = k - 1;
                    const int st = j & 1;
                    if (!mbar_wait(p_full + st, (j >> 1) & 1, abort_flag, ERR_SITE_PREFILL | 5)) break;
                    if (!mbar_wait(v_full + st, (j >> 1) & 1, abort_flag, ERR_SITE_PREFILL | 6)) break;
                    tc_fence_after();
                    const uint32_t v_base = smem_u32(smem + OFF_V + st * V_STAGE_BYTES);
                    const uint32_t p_tmem = tmem + S_COL0 + st * 128;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        umma_ts(tmem + O_COL, p_tmem + kk * 8, desc_sw128(v_base + kk * 2048, K_CHUNK_BYTES, 1024),
                                idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(o_done);
                    umma_commit(v_empty + st);
                    if (j == n_tiles - 1) umma_commit(o_final);
                }
            }
        }
    } else {
        // --------------------------- softmax + epilogue ---------------------------
        const int r = warp * 32 + lane;  // TMEM lane == tile row
        const bool is_sig = r < SIG_ROWS;
        const bool is_noise = (r >= NOISE_ROW0) && (r < NOISE_ROW0 + TOK);
        const int tau = is_sig ? (r >> 2) : (r - NOISE_ROW0);
        const int t = t0 + tau;
        const int lo_t = (window > 0) ? t - window + 1 : -0x40000000;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float c_log2 = 0.07216878364870322f * 1.4426950408889634f;  // log2(e) / sqrt(192)
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;

        for (int k = 0; k < n_tiles; ++k) {
            const int st = k & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(s_full + st, (k >> 1) & 1, abort_flag, ERR_SITE_PREFILL | 7))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t s_addr = lane_base + S_COL0 + st * 128;
            float s[BN];
            {
                uint32_t rr[64];
                tmem_ld64(s_addr, rr);
#pragma unroll
                for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(rr[i]);
                tmem_ld64(s_addr + 64, rr);
#pragma unroll
                for (int i = 0; i < 64; ++i) s[64 + i] = __uint_as_float(rr[i]);
            }
            const int u0 = kv_lo + k * BN;
            const bool need_mask = (u0 + BN - 1 > t0) || (window > 0 && u0 < t0 + TOK - window);
            if (need_mask) {
#pragma unroll
                for (int i = 0; i < BN; ++i) {
                    const int u = u0 + i;
                    if (u > t || u < lo_t) s[i] = -INFINITY;
                }
            }
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int i = 4; i < BN; i += 4) {
                mx0 = fmaxf(mx0, s[i]);
                mx1 = fmaxf(mx1, s[i + 1]);
                mx2 = fmaxf(mx2, s[i + 2]);
                mx3 = fmaxf(mx3, s[i + 3]);
            }
            const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c_log2;
            const float m_new = fmaxf(m_run, mx);
            float alpha = 1.f;
            bool resc = false;
            if (m_new > m_run + kRescaleThreshold) {
                alpha = fast_exp2(m_run - m_new);
                l_run *= alpha;
                m_run = m_new;
                resc = true;
            }
            const float mb = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pk[BN / 2];
            float l0 = 0.f, l1 = 0.f;
#pragma unroll
            for (int i = 0; i < BN; i += 2) {
                const float p0 = fast_exp2(fmaf(s[i], c_log2, -mb));
                const float p1 = fast_exp2(fmaf(s[i + 1], c_log2, -mb));
                l0 += p0;
                l1 += p1;
                pk[i >> 1] = pack_bf16x2(p0, p1);
            }
            l_run += l0 + l1;
            if (k > 0 && __any_sync(0xffffffffu, resc)) {
                if (!__all_sync(0xffffffffu, mbar_wait(o_done, (k - 1) & 1, abort_flag, ERR_SITE_PREFILL | 8))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float a = resc ? alpha : 1.f;
#pragma unroll
                for (int ch = 0; ch < DV / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + O_COL + ch * 32, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                    tmem_st32(lane_base + O_COL + ch * 32, o);
                }
            }
            {
                uint32_t (&p0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&pk[0]);
                uint32_t (&p1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&pk[32]);
                tmem_st32(s_addr, p0);
                tmem_st32(s_addr + 32, p1);
            }
            tc_fence_before();
            mbar_arrive(p_full + st);
        }

        // ------------------------------- epilogue --------------------------------
        // o_done may still be two phases behind here, which a parity wait cannot
        // tell apart; o_final completes exactly once, after the last PV product.
        if (ok && !mbar_wait(o_final, 0, abort_flag, ERR_SITE_PREFILL | 9)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
        float *hn = reinterpret_cast<float *>(smem + OFF_K);  // K stage 0 is free once every MMA is done
        if (warp == 3) {
#pragma unroll
            for (int ch = 0; ch < DV / 32; ++ch) {
                uint32_t o[32];
                tmem_ld32(lane_base + O_COL + ch * 32, o);
                if (is_noise) {
                    float4 *dst = reinterpret_cast<float4 *>(hn + tau * HN_STRIDE + ch * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                             __uint_as_float(o[4 * i + 2]) * inv_l,
                                             __uint_as_float(o[4 * i + 3]) * inv_l);
                }
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (warp < 3) {
            const bool valid = ok && (t < L);
            const int n_idx = s0 + t;
            const int head = 4 * group + (r & 3);
            const size_t row = static_cast<size_t>(n_idx) * hs + head;
            const float lam = valid ? lambda[row] : 0.f;
            const uint4 *g_row = reinterpret_cast<const uint4 *>(gate + row * DV);
            uint4 *o_row = reinterpret_cast<uint4 *>(out + row * DV);
            const float *hn_row = hn + tau * HN_STRIDE;
#pragma unroll
            for (int ch = 0; ch < DV / 32; ++ch) {
                uint32_t o[32];
                tmem_ld32(lane_base + O_COL + ch * 32, o);
                if (valid) {
                    uint4 gv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) gv[i] = __ldg(g_row + ch * 4 + i);
                    const uint32_t *gw = reinterpret_cast<const uint32_t *>(gv);
                    uint32_t res[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gw[i]));
                        const float d0 = __uint_as_float(o[2 * i]) * inv_l - lam * hn_row[ch * 32 + 2 * i];
                        const float d1 = __uint_as_float(o[2 * i + 1]) * inv_l - lam * hn_row[ch * 32 + 2 * i + 1];
                        const float y0 = __fdividef(d0, 1.f + __expf(-g2.x));
                        const float y1 = __fdividef(d1, 1.f + __expf(-g2.y));
                        res[i] = pack_bf16x2(y0, y1);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        o_row[ch * 4 + i] = make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, pf::TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------
int prefill_smem_bytes() { return pf::SMEM_BYTES; }

cudaError_t launch_prefill(const PrefillLaunch &L, const PrefillPlan &plan, cudaStream_t stream) {
    static_assert(pf::SMEM_BYTES <= 232448, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(gdla_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         pf::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>(plan.n_items) * static_cast<unsigned>(plan.hkv);
    gdla_prefill_kernel<<<grid, pf::NUM_THREADS, pf::SMEM_BYTES, stream>>>(
        L.tm_qs, L.tm_qn, L.tm_k, L.tm_v, L.lambda, L.gate, L.out, plan);
    return cudaPeekAtLastError();
}

}  // namespace gdla
