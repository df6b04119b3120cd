// gdla_decode_latent.cu - GDLA decode over the compressed (latent) KV cache,
// with the key and value up-projections absorbed, for sm_100a.
//
// Method (aitrends.kr/articles/94908, head-configuration paragraph: KV
// low-rank dimension 512 and one rotary key of 64 shared by every KV head;
// the 16 KV heads are an up-projection of that compressed row; the paragraph
// on MLA's compressed KV cache for decoding). Per token the cache holds one
// 576-wide row [c (512) | k_rope (64)]. With the non-rotary query part
// absorbed into W^UK_j (q_abs = [W^UK_j^T q_nope | q_rope], prepared by the
// caller), every query head of every group scores the same rows:
//     s_u = q_abs . [c_u | kr_u] / sqrt(192)
// and its output is H = W^UV_j (sum_u p_u c_u) / (sum_u p_u), W^UV_j [128 x 512];
// then D_i = H_S,i - lambda_i H_N,j and out_i = sigmoid(gate_i) D_i.
//
// Split kernel (one CTA per (sequence, split) item, all 5*hkv heads at once):
//   S   = Q C^T        tcgen05 M=128 (query heads, up to 80 live rows) N=48 keys
//                      K=576; Q and a 48-key stage of C in shared memory
//   softmax            one TMEM lane (thread) per head row, online max/sum
//   O^T += C_lat^T P^T tcgen05 M=128 (latent dims, 4 blocks) N=heads K=48 keys:
//                      A = the same C stage read dims-major, B = P (bf16,
//                      written to shared memory by the softmax threads)
// Keeping the latent dims as the M of the second product puts O^T (512 dims x
// 80 heads fp32) in 320 TMEM columns; with heads as M it would need all 512.
// A 48-key stage (54 KB) is what two stages leave room for beside the 90 KB of
// queries. The item's unnormalised O, its running max and sum go to the
// workspace; the combine kernel merges the splits, applies W^UV_j and the
// GDLA epilogue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

namespace lt {
constexpr int DC = 512, DR = 64, DL = DC + DR, DQK = 192, DV = 128;
constexpr int LCH = DL / 64;             // 9 chunks of 64 dims
constexpr int TK = 48;                   // keys per stage
constexpr int STAGES = 2;
constexpr int MAX_ROWS = 80;             // query head rows per CTA (hkv <= 16)
constexpr int Q_CH = MAX_ROWS * 128;     // one 64-dim chunk of Q: 80 rows x 128 B
constexpr int C_CH = TK * 128;           // one 64-dim chunk of a stage: 48 keys x 128 B
constexpr int C_STAGE = LCH * C_CH;      // 55,296 B
constexpr int P_BUF = MAX_ROWS * 128;    // P rows (keys 0..47 of 64) per head row
constexpr int OFF_Q = 0;
// An M=128 MMA reads 128 A rows: the 48 rows past the 80 of a chunk fall in
// the next chunk (after the last chunk: in the P buffers). Their S rows are
// never used.
constexpr int OFF_P = OFF_Q + LCH * Q_CH;
constexpr int OFF_C = OFF_P + 2 * P_BUF;
constexpr int OFF_BAR = OFF_C + STAGES * C_STAGE;
constexpr int OFF_ML = OFF_BAR + 16 * 8;        // per head row: this item's alpha (rescale), flag
constexpr int OFF_MISC = OFF_ML + 128 * 4 + 16;
constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
constexpr uint32_t O_BLK = 80;           // TMEM columns per 128-dim block of O^T
constexpr uint32_t S_COL0 = 4 * O_BLK;   // 320; two S buffers of TK columns
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr int NUM_THREADS = 128 + 64;    // 4 softmax/epilogue warps, producer, MMA
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(S_COL0 + 2 * TK <= TMEM_COLS, "TMEM budget");
}  // namespace lt

// Rows of the head layout in Q / S / P: signal heads 0..4H-1 at rows 0..4H-1,
// noise heads at rows NS_PAD..NS_PAD+H-1 (NS_PAD = 4H rounded up to 8, so the
// noise TMA box lands on a 1024-byte swizzle-atom boundary).
__host__ __device__ constexpr int latent_ns_pad(int hkv) { return (4 * hkv + 7) / 8 * 8; }
__host__ __device__ constexpr int latent_rows(int hkv) { return latent_ns_pad(hkv) + hkv; }
// N of the O^T MMA: the used rows rounded up to 16.
__host__ __device__ constexpr int latent_n(int hkv) { return (latent_rows(hkv) + 15) / 16 * 16; }

// OR of `v` over the 128 softmax threads (named barrier 1).
__device__ __forceinline__ bool bar_or_128(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v))
        : "memory");
    return r != 0;
}

struct LatentItem {
    int b, split, start, k_begin, k_end, n_stages;
};

__device__ __forceinline__ LatentItem latent_item(const int32_t *__restrict__ cu, int w, const LatentPlan &plan) {
    LatentItem d;
    d.split = w % plan.num_splits;
    d.b = w / plan.num_splits;
    d.start = cu[d.b];
    const int end = cu[d.b + 1];
    const int len = end - d.start;
    const bool ok = (d.start >= 0) && (len >= 1) && (len <= plan.max_seqlen_k) && (end <= plan.num_cache_rows);
    const int lo = (plan.window > 0) ? max(0, len - plan.window) : 0;
    const int n_vis = ok ? len - lo : 0;
    d.k_begin = lo + d.split * plan.split_keys;
    d.k_end = lo + min(n_vis, (d.split + 1) * plan.split_keys);
    d.n_stages = max(0, (d.k_end - d.k_begin + lt::TK - 1) / lt::TK);
    return d;
}

__global__ void __launch_bounds__(lt::NUM_THREADS, 1)
gdla_decode_latent_split_kernel(const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_qn,
                                const __grid_constant__ CUtensorMap tm_c, const int32_t *__restrict__ cu_seqlens_k,
                                float *__restrict__ ws, const LatentPlan plan) {
    using namespace lt;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *q_full = bars + 0;
    uint64_t *c_full = bars + 1;    // [stage]
    uint64_t *c_empty = bars + 3;   // [stage]
    uint64_t *s_full = bars + 5;    // [buffer]
    uint64_t *p_full = bars + 7;    // [buffer]
    uint64_t *o_done = bars + 9;    // one phase per O^T product
    uint64_t *o_final = bars + 10;  // the item's last O^T product is done
    float *alpha_s = reinterpret_cast<float *>(smem + OFF_ML);  // [128]: per head row rescale of O^T
    int *resc_flag = reinterpret_cast<int *>(smem + OFF_ML + 128 * 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hkv = plan.hkv;
    const int ns_pad = latent_ns_pad(hkv);
    const int w = blockIdx.x;  // one item per CTA
    const LatentItem it = latent_item(cu_seqlens_k, w, plan);
    const int nst = it.n_stages;
    const size_t slot = static_cast<size_t>(w);  // (b * num_splits + split)

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(c_full + i, 1);
            mbar_init(c_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full + i, 1);
            mbar_init(p_full + i, 128);
        }
        mbar_init(o_done, 1);
        mbar_init(o_final, 1);
        *abort_flag = 0;
        *resc_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (nst > 0) {
        if (warp == 4) {
            // ------------------------------ TMA producer ------------------------------
            if (lane == 0) {
                tma_prefetch_desc(&tm_c);
                mbar_arrive_expect_tx(q_full, LCH * (4 * hkv + hkv) * 128);
                for (int c = 0; c < LCH; ++c) {
                    tma_load_3d(smem + OFF_Q + c * Q_CH, &tm_qs, q_full, c * 64, 0, it.b);
                    tma_load_3d(smem + OFF_Q + c * Q_CH + ns_pad * 128, &tm_qn, q_full, c * 64, 0, it.b);
                }
                int issued = 0;
                for (int k = 0; k < nst; ++k) {
                    const int st = k % STAGES;
                    if (k >= STAGES &&
                        !mbar_wait(c_empty + st, ((k / STAGES) + 1) & 1, abort_flag, ERR_SITE_LATENT | 1))
                        break;
                    mbar_arrive_expect_tx(c_full + st, C_STAGE);
                    const int row = it.start + it.k_begin + k * TK;
                    for (int c = 0; c < LCH; ++c)
                        tma_load_3d(smem + OFF_C + st * C_STAGE + c * C_CH, &tm_c, c_full + st, c * 64, 0, row);
                    issued = k + 1;
                }
                if (*abort_flag) {
                    for (int k = max(0, issued - STAGES); k < issued; ++k)
                        mbar_wait_cycles(c_full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
                    mbar_wait_cycles(q_full, 0, 1ll << 22);
                }
            }
        } else if (warp == 5) {
            // ------------------------------ MMA issuer --------------------------------
            // Order: S(0), S(1), then per stage k: O^T(k) (after P(k)), S(k+2).
            // S(k+2) reuses S buffer k&1 and the P buffer of stage k is next
            // written for stage k+2, whose s_full commit follows O^T(k).
            const uint32_t leader = elect_one_sync();
            const int n_mma = latent_n(hkv);
            const uint32_t idesc_s = idesc_bf16_f32(128, TK, false, false);
            const uint32_t idesc_o = idesc_bf16_f32(128, n_mma, true, false);
            const uint64_t q_desc0 = desc_sw128(smem_u32(smem + OFF_Q), 16, 1024);
            const uint64_t c_desc0 = desc_sw128(smem_u32(smem + OFF_C), 16, 1024);      // C as B (keys x dims)
            const uint64_t ct_desc0 = desc_sw128(smem_u32(smem + OFF_C), C_CH, 1024);   // C as A (dims-major)
            const uint64_t p_desc0 = desc_sw128(smem_u32(smem + OFF_P), 16, 1024);
            bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, ERR_SITE_LATENT | 2));
            auto issue_s = [&](int k) {
                const int st = k % STAGES;
                if (!__all_sync(0xffffffffu, mbar_wait(c_full + st, (k / STAGES) & 1, abort_flag, ERR_SITE_LATENT | 3)))
                    return false;
                tc_fence_after();
                const uint32_t d = tmem + S_COL0 + (k & 1) * TK;
#pragma unroll
                for (int kk = 0; kk < DL / 16; ++kk) {
                    const uint32_t offq = ((kk >> 2) * Q_CH + (kk & 3) * 32) >> 4;
                    const uint32_t offc = (st * C_STAGE + (kk >> 2) * C_CH + (kk & 3) * 32) >> 4;
                    umma_ss_leader(d, q_desc0 + offq, c_desc0 + offc, idesc_s, kk > 0, leader);
                }
                umma_commit_leader(s_full + (k & 1), leader);
                return true;
            };
            for (int k = 0; ok && k < min(2, nst); ++k) ok = issue_s(k);
            for (int k = 0; ok && k < nst; ++k) {
                const int st = k % STAGES;
                if (!__all_sync(0xffffffffu, mbar_wait(p_full + (k & 1), (k >> 1) & 1, abort_flag, ERR_SITE_LATENT | 4))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // O^T[dims 128m..128m+127][heads] += C_lat^T[dims][keys] P^T[keys][heads]
#pragma unroll
                for (int m = 0; m < DC / 128; ++m)
#pragma unroll
                    for (int ks = 0; ks < TK / 16; ++ks) {
                        const uint32_t offa = (st * C_STAGE + 2 * m * C_CH + ks * 2048) >> 4;
                        const uint32_t offb = ((k & 1) * P_BUF + ks * 32) >> 4;
                        umma_ss_leader(tmem + m * O_BLK, ct_desc0 + offa, p_desc0 + offb, idesc_o,
                                       (k > 0 || ks > 0) ? 1u : 0u, leader);
                    }
                umma_commit_leader(o_done, leader);
                umma_commit_leader(c_empty + st, leader);
                if (k == nst - 1) umma_commit_leader(o_final, leader);
                if (k + 2 < nst) ok = issue_s(k + 2);
            }
        } else {
            // --------------------------- softmax + epilogue ---------------------------
            // Thread = head row r (TMEM lane r of S, P row r). Rows < 4H: signal
            // heads; rows ns_pad .. ns_pad+H-1: noise heads; others unused.
            const int r = threadIdx.x;
            // rows that hold a query head (the others hold whatever the MMA read there)
            const bool real = (r < 4 * hkv) || (r >= ns_pad && r < ns_pad + hkv);
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            const float c_log2 = 0.07216878364870322f * 1.4426950408889634f;  // log2(e) / sqrt(192)
            float m_run = -INFINITY, l_run = 0.f;
            uint8_t *p_row0 = smem + OFF_P + (r >> 3) * 1024 + (r & 7) * 128;
            bool ok = true;
            for (int k = 0; k < nst; ++k) {
                const int b2 = k & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(s_full + b2, (k >> 1) & 1, abort_flag, ERR_SITE_LATENT | 5))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float s[TK];
                {
                    uint32_t ra[32], rb[16];
                    tmem_ld32(lane_base + S_COL0 + b2 * TK, ra);
                    tmem_ld16(lane_base + S_COL0 + b2 * TK + 32, rb);
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[i] = __uint_as_float(ra[i]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) s[32 + i] = __uint_as_float(rb[i]);
                }
                const int u0 = it.k_begin + k * TK;
                if (u0 + TK > it.k_end) {
#pragma unroll
                    for (int i = 0; i < TK; ++i)
                        if (u0 + i >= it.k_end) s[i] = -INFINITY;
                }
                float mx = s[0];
#pragma unroll
                for (int i = 1; i < TK; ++i) mx = fmaxf(mx, s[i]);
                mx *= c_log2;
                // lazy rescale: O^T column r is rescaled only when the max grows by > 2^8
                float alpha = 1.f;
                bool resc = false;
                if (real && mx > m_run + kRescaleThreshold) {
                    alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - mx);
                    l_run *= alpha;
                    resc = (k > 0);
                    m_run = mx;
                }
                const float mb = (m_run == -INFINITY) ? 0.f : m_run;
                uint32_t pk[TK / 2];
                float lsum = 0.f;
#pragma unroll
                for (int i = 0; i < TK / 2; ++i) {
                    const float p0 = fast_exp2(fmaf(s[2 * i], c_log2, -mb));
                    const float p1 = fast_exp2(fmaf(s[2 * i + 1], c_log2, -mb));
                    lsum += p0 + p1;
                    pk[i] = real ? pack_bf16x2(p0, p1) : 0u;
                }
                l_run += lsum;
                // P row r of buffer b2 (K-major, 128-byte swizzle): keys 0..47 = units 0..5
                if (r < MAX_ROWS) {
                    uint8_t *prow = p_row0 + b2 * P_BUF;
#pragma unroll
                    for (int u = 0; u < TK / 8; ++u)
                        *reinterpret_cast<uint4 *>(prow + ((u ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                }
                fence_proxy_async_smem();
                // O^T columns of rescaled heads: every thread (as a dims lane of
                // O^T) scales them once the previous O^T product is done.
                if (bar_or_128(resc)) {
                    alpha_s[r] = resc ? alpha : 1.f;
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (!__all_sync(0xffffffffu, mbar_wait(o_done, (k - 1) & 1, abort_flag, ERR_SITE_LATENT | 6))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int n_cols = latent_n(hkv);
                    for (int m = 0; m < DC / 128; ++m)
                        for (int c0 = 0; c0 < n_cols; c0 += 16) {
                            uint32_t o[16];
                            tmem_ld16(lane_base + m * O_BLK + c0, o);
#pragma unroll
                            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha_s[c0 + i]);
                            tmem_st16(lane_base + m * O_BLK + c0, o);
                        }
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                }
                tc_fence_before();
                mbar_arrive(p_full + b2);
            }
            if (ok && __all_sync(0xffffffffu, mbar_wait(o_final, 0, abort_flag, ERR_SITE_LATENT | 7))) {
                tc_fence_after();
                // Split partial: O (unnormalised, per head row and latent dim), m, l.
                const int rows = latent_rows(hkv);
                float *wo = ws + slot * (static_cast<size_t>(MAX_ROWS) * DC);
                for (int m = 0; m < DC / 128; ++m)
                    for (int c0 = 0; c0 < rows; c0 += 16) {
                        uint32_t o[16];
                        tmem_ld16(lane_base + m * O_BLK + c0, o);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < rows) wo[(c0 + i) * DC + m * 128 + r] = __uint_as_float(o[i]);
                    }
                if (r < rows) {
                    float *wml = ws + plan.ml_offset_floats + slot * (MAX_ROWS * 2);
                    wml[2 * r] = m_run;
                    wml[2 * r + 1] = l_run;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Combine: one CTA per (group j, block of BB sequences). It merges each
// sequence's splits of the group's 5 head rows (log-sum-exp weights) into
// o [BB x 5 x 512] fp32, then forms H = W^UV_j o on the tensor cores:
//     D [128 dims x 80] = W^UV_j [128 x 512] . B^T,  B [80 x 512]
// with B's rows (sequence, head, part): part 0 the bf16 rounding of o, part 1
// the bf16 rounding of the remainder, so that the product carries o to about
// 16 bits (one bf16 rounding alone would leave ~1e-3 relative error in H,
// which D = H_S - lambda H_N can magnify). W^UV_j (128 KB) comes in by TMA
// once per BB sequences; warps 0-3 (one TMEM lane = one output dim each) add
// the parts and apply the GDLA epilogue.
namespace lc {
constexpr int BB = 8;                  // sequences per CTA
constexpr int NCOMBO = BB * 5;         // (sequence, head) rows of o
constexpr int NR = 2 * NCOMBO;         // B rows: 80
constexpr int W_CH = 128 * 128;        // a 64-dim chunk of W^UV_j: 128 rows x 128 B
constexpr int B_CH = NR * 128;         // a 64-dim chunk of B: 80 rows x 128 B
constexpr int OFF_W = 0;
constexpr int OFF_B = OFF_W + 8 * W_CH;
constexpr int OFF_WGT = OFF_B + 8 * B_CH;                 // [NCOMBO][kLatentMaxSplits] merge weights
constexpr int OFF_INVL = OFF_WGT + NCOMBO * kLatentMaxSplits * 4;
constexpr int OFF_NSB = OFF_INVL + NCOMBO * 4;           // [BB] splits of each sequence
constexpr int OFF_BAR = OFF_NSB + BB * 4;
constexpr int OFF_MISC = OFF_BAR + 2 * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int NUM_THREADS = 256;
constexpr uint32_t TMEM_COLS = 128;
static_assert(OFF_B % 1024 == 0 && B_CH % 1024 == 0, "swizzle atoms");
static_assert(OFF_BAR % 8 == 0, "barrier alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace lc

__global__ void __launch_bounds__(lc::NUM_THREADS, 1)
gdla_decode_latent_combine_kernel(const __grid_constant__ CUtensorMap tm_w, const float *__restrict__ ws,
                                  const int32_t *__restrict__ cu_seqlens_k, const float *__restrict__ lambda,
                                  const __nv_bfloat16 *__restrict__ gate, __nv_bfloat16 *__restrict__ out,
                                  const LatentPlan plan) {
    using namespace lc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *wgt_s = reinterpret_cast<float *>(smem + OFF_WGT);
    float *inv_l_s = reinterpret_cast<float *>(smem + OFF_INVL);
    int *nsb_s = reinterpret_cast<int *>(smem + OFF_NSB);
    uint64_t *w_full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *mma_done = w_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    const int j = blockIdx.x, b0 = blockIdx.y * BB;
    const int hkv = plan.hkv, ns = plan.num_splits, batch = plan.batch;
    const int ns_pad = latent_ns_pad(hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *wml = ws + plan.ml_offset_floats;

    if (threadIdx.x == 0) {
        mbar_init(w_full, 1);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(w_full, 8 * W_CH);
        for (int c = 0; c < 8; ++c) tma_load_3d(smem + OFF_W + c * W_CH, &tm_w, w_full, c * 64, 0, j);
    }

    // Splits holding keys of each sequence of the block (the split kernel wrote
    // the others nothing); 0 past the batch.
    if (threadIdx.x < BB) {
        const int b = b0 + threadIdx.x;
        int n = 0;
        if (b < batch) {
            const int start = cu_seqlens_k[b], end = cu_seqlens_k[b + 1];
            const int len = end - start;
            const bool valid =
                (start >= 0) && (len >= 1) && (len <= plan.max_seqlen_k) && (end <= plan.num_cache_rows);
            const int lo = (plan.window > 0) ? max(0, len - plan.window) : 0;
            const int n_vis = valid ? len - lo : 0;
            n = min(ns, (n_vis + plan.split_keys - 1) / plan.split_keys);
        }
        nsb_s[threadIdx.x] = n;
    }
    // Epilogue operands (warps 0-3: output dim d = threadIdx.x), loaded while the
    // rest runs: gate logit and lambda of each (sequence, signal head).
    uint32_t g_pre[BB * 4 / 2];  // bf16 pairs
    float lam_pre[BB * 4];
    if (warp < 4) {
#pragma unroll
        for (int sl = 0; sl < BB; ++sl)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int b = min(b0 + sl, batch - 1);
                const size_t orow = static_cast<size_t>(b) * 4 * hkv + 4 * j + i;
                const uint16_t gv = __ldg(reinterpret_cast<const unsigned short *>(gate) + orow * lt::DV + threadIdx.x);
                if (i & 1)
                    g_pre[sl * 2 + (i >> 1)] |= static_cast<uint32_t>(gv) << 16;
                else
                    g_pre[sl * 2 + (i >> 1)] = gv;
                lam_pre[sl * 4 + i] = __ldg(lambda + orow);
            }
    }
    __syncthreads();
    // Merge weights: warp w takes combos w, w + 8, ... (all loads first); lane = split (ns <= 32).
    {
        constexpr int PER_WARP = NCOMBO / (NUM_THREADS / 32);
        static_assert(NCOMBO % (NUM_THREADS / 32) == 0, "combos per warp");
        float ms[PER_WARP], ls[PER_WARP];
#pragma unroll
        for (int q = 0; q < PER_WARP; ++q) {
            const int c = warp + q * (NUM_THREADS / 32);
            const int hh = c % 5;
            const int row = (hh < 4) ? 4 * j + hh : ns_pad + j;
            const bool mine = lane < nsb_s[c / 5];
            const size_t base = (static_cast<size_t>(b0 + c / 5) * ns + lane) * (lt::MAX_ROWS * 2) + 2 * row;
            ms[q] = mine ? wml[base] : -INFINITY;
            ls[q] = mine ? wml[base + 1] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < PER_WARP; ++q) {
            const int c = warp + q * (NUM_THREADS / 32);
            float M = ms[q];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
            const float wgt = (ms[q] == -INFINITY) ? 0.f : fast_exp2(ms[q] - M);
            float L = ls[q] * wgt;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
            wgt_s[c * kLatentMaxSplits + lane] = wgt;
            if (lane == 0) inv_l_s[c] = (L > 0.f) ? 1.f / L : 0.f;
        }
    }
    __syncthreads();
    // B rows 2c (bf16 of o) and 2c+1 (bf16 of the remainder), K-major with the
    // 128-byte swizzle: task = (combo c, 8-dim unit u of 64). Every thread's
    // tasks load their first split together, then the remaining splits.
    {
        constexpr int TASKS = NCOMBO * 64 / NUM_THREADS;  // 10
        static_assert((NCOMBO * 64) % NUM_THREADS == 0, "tasks per thread");
        float acc[TASKS][8];
        auto src_of = [&](int q, int sp) {
            const int task = threadIdx.x + q * NUM_THREADS;
            const int c = task >> 6, u = task & 63;
            const int hh = c % 5;
            const int row = (hh < 4) ? 4 * j + hh : ns_pad + j;
            return reinterpret_cast<const float4 *>(
                ws + ((static_cast<size_t>(b0 + c / 5) * ns + sp) * lt::MAX_ROWS + row) * lt::DC + u * 8);
        };
#pragma unroll
        for (int q = 0; q < TASKS; ++q) {
            const int c = (threadIdx.x + q * NUM_THREADS) >> 6;
            float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
            if (nsb_s[c / 5] > 0) {
                const float4 *src = src_of(q, 0);
                x0 = __ldg(src);
                x1 = __ldg(src + 1);
            }
            const float wgt = wgt_s[c * kLatentMaxSplits];
            acc[q][0] = wgt * x0.x;
            acc[q][1] = wgt * x0.y;
            acc[q][2] = wgt * x0.z;
            acc[q][3] = wgt * x0.w;
            acc[q][4] = wgt * x1.x;
            acc[q][5] = wgt * x1.y;
            acc[q][6] = wgt * x1.z;
            acc[q][7] = wgt * x1.w;
        }
        int ns_max = 0;
#pragma unroll
        for (int sl = 0; sl < BB; ++sl) ns_max = max(ns_max, nsb_s[sl]);
        for (int sp = 1; sp < ns_max; ++sp) {
#pragma unroll
            for (int q = 0; q < TASKS; ++q) {
                const int c = (threadIdx.x + q * NUM_THREADS) >> 6;
                const float wgt = wgt_s[c * kLatentMaxSplits + sp];
                if (sp >= nsb_s[c / 5] || wgt == 0.f) continue;
                const float4 *src = src_of(q, sp);
                const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
                acc[q][0] = fmaf(wgt, x0.x, acc[q][0]);
                acc[q][1] = fmaf(wgt, x0.y, acc[q][1]);
                acc[q][2] = fmaf(wgt, x0.z, acc[q][2]);
                acc[q][3] = fmaf(wgt, x0.w, acc[q][3]);
                acc[q][4] = fmaf(wgt, x1.x, acc[q][4]);
                acc[q][5] = fmaf(wgt, x1.y, acc[q][5]);
                acc[q][6] = fmaf(wgt, x1.z, acc[q][6]);
                acc[q][7] = fmaf(wgt, x1.w, acc[q][7]);
            }
        }
#pragma unroll
        for (int q = 0; q < TASKS; ++q) {
            const int task = threadIdx.x + q * NUM_THREADS;
            const int c = task >> 6, u = task & 63;
            const float il = inv_l_s[c];
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float v0 = acc[q][2 * i] * il, v1 = acc[q][2 * i + 1] * il;
                hi[i] = pack_bf16x2(v0, v1);
                const float h0 = __uint_as_float(hi[i] << 16), h1 = __uint_as_float(hi[i] & 0xFFFF0000u);
                lo[i] = pack_bf16x2(v0 - h0, v1 - h1);
            }
            const int kc = u >> 3, unit = u & 7;
            uint8_t *chunk = smem + OFF_B + kc * B_CH;
            const int r0 = 2 * c, r1 = 2 * c + 1;
            *reinterpret_cast<uint4 *>(chunk + r0 * 128 + ((unit ^ (r0 & 7)) << 4)) =
                make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(chunk + r1 * 128 + ((unit ^ (r1 & 7)) << 4)) =
                make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        const uint32_t leader = elect_one_sync();
        const bool ok = __all_sync(0xffffffffu, mbar_wait(w_full, 0, abort_flag, ERR_SITE_LATENT | 8));
        if (ok) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(128, NR, false, false);
            const uint64_t w_desc0 = desc_sw128(smem_u32(smem + OFF_W), 16, 1024);
            const uint64_t b_desc0 = desc_sw128(smem_u32(smem + OFF_B), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < lt::DC / 16; ++kk) {
                const uint32_t offw = ((kk >> 2) * W_CH + (kk & 3) * 32) >> 4;
                const uint32_t offb = ((kk >> 2) * B_CH + (kk & 3) * 32) >> 4;
                umma_ss_leader(tmem, w_desc0 + offw, b_desc0 + offb, idesc, kk > 0, leader);
            }
            umma_commit_leader(mma_done, leader);
        } else if (lane == 0) {
            mbar_wait_cycles(w_full, 0, 1ll << 22);  // the W^UV copy lands before the CTA leaves
        }
    }
    if (warp < 4) {
        // Thread = output dim d (TMEM lane); columns 10 s' + 2 hh + part.
        const bool ok = __all_sync(0xffffffffu, mbar_wait(mma_done, 0, abort_flag, ERR_SITE_LATENT | 9));
        if (ok) {
            tc_fence_after();
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            uint32_t ra[32], rb[32], rc[16];
            tmem_ld32(lane_base, ra);
            tmem_ld32(lane_base + 32, rb);
            tmem_ld16(lane_base + 64, rc);
            auto col = [&](int n) -> float {
                return __uint_as_float(n < 32 ? ra[n] : (n < 64 ? rb[n - 32] : rc[n - 64]));
            };
            const int d = threadIdx.x;
#pragma unroll
            for (int sl = 0; sl < BB; ++sl) {
                const int b = b0 + sl;
                if (b >= batch) break;
                const float hn = col(10 * sl + 8) + col(10 * sl + 9);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float hsig = col(10 * sl + 2 * i) + col(10 * sl + 2 * i + 1);
                    const size_t orow = static_cast<size_t>(b) * 4 * hkv + 4 * j + i;
                    const float dd = hsig - lam_pre[sl * 4 + i] * hn;
                    const uint32_t gp = g_pre[sl * 2 + (i >> 1)];
                    const float g = __uint_as_float((i & 1) ? (gp & 0xFFFF0000u) : (gp << 16));
                    out[orow * lt::DV + d] = __float2bfloat16_rn(__fdividef(dd, 1.f + __expf(-g)));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

LatentPlan make_latent_plan(int batch, int hkv, int max_seqlen_k, int window, int num_cache_rows) {
    LatentPlan p{};
    p.batch = batch;
    p.hkv = hkv;
    p.window = window;
    p.max_seqlen_k = max_seqlen_k;
    p.num_cache_rows = num_cache_rows;
    const int eff = (window > 0) ? (window < max_seqlen_k ? window : max_seqlen_k) : max_seqlen_k;
    int ns = (eff + kLatentMinSplitKeys - 1) / kLatentMinSplitKeys;
    ns = ns < 1 ? 1 : (ns > kLatentMaxSplits ? kLatentMaxSplits : ns);
    int keys = (eff + ns - 1) / ns;
    keys = (keys + lt::TK - 1) / lt::TK * lt::TK;
    p.split_keys = keys;
    p.num_splits = (eff + keys - 1) / keys;
    p.ml_offset_floats = static_cast<long long>(batch) * p.num_splits * lt::MAX_ROWS * lt::DC;
    return p;
}

size_t latent_workspace_bytes(const LatentPlan &p) {
    return static_cast<size_t>(p.batch) * p.num_splits * lt::MAX_ROWS * (lt::DC + 2) * sizeof(float);
}

cudaError_t launch_decode_latent(const LatentLaunch &L, const LatentPlan &plan, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static PerContextFlag attr_set;
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        e = cudaFuncSetAttribute(gdla_decode_latent_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 lt::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    const unsigned items = static_cast<unsigned>(plan.batch * plan.num_splits);
    gdla_decode_latent_split_kernel<<<items, lt::NUM_THREADS, lt::SMEM_BYTES, stream>>>(L.tm_qs, L.tm_qn, L.tm_c,
                                                                                       L.cu_seqlens_k, L.ws, plan);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    static PerContextFlag combine_attr_set;
    if (!combine_attr_set.is_set(dev, ctx)) {
        e = cudaFuncSetAttribute(gdla_decode_latent_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 lc::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        combine_attr_set.set(dev, current_context_id());
    }
    dim3 grid2(plan.hkv, (plan.batch + lc::BB - 1) / lc::BB);
    gdla_decode_latent_combine_kernel<<<grid2, lc::NUM_THREADS, lc::SMEM_BYTES, stream>>>(
        L.tm_w, L.ws, L.cu_seqlens_k, L.lambda, L.gate, L.out, plan);
    return cudaPeekAtLastError();
}

}  // namespace gdla
