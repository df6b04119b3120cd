// gdla_decode.cu - varlen split-KV GDLA decode for sm_100a.
//
// One query token per sequence (position L_b - 1, the cache holding it). For
// each (sequence b, KV group j, split s) item a persistent CTA streams the
// split's slice of K_j/V_j through shared memory (TMA, 64 keys per stage; the
// stage ring continues across items) and computes, for the five
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

#include <atomic>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

namespace dc {
constexpr int DQK = 192, DV = 128, HEADS = 5;
constexpr int STAGES = 2;
// Per-stage auxiliary area. The producer writes the item's key range into
// every stage it issues and, with an item's first stage, bulk-copies the
// item's queries (and, when one split holds every key, its gate logits and
// lambda) there, so the consumers never wait on global loads of their own.
constexpr int Q_ROW = DQK * 2;                      // 384 bytes per query row
constexpr int Q_ROW_STRIDE = Q_ROW + 16;            // padded: ldmatrix rows fall in distinct banks
constexpr int AUX_DESC = 0;                         // int[4]: first cache row, k_begin, k_end, n_stages
constexpr int AUX_LAM = 16;                         // fp32[4]
constexpr int AUX_Q = 128;                          // bf16 [8 rows: 4 signal, noise, 3 zero][Q_ROW_STRIDE]
constexpr int AUX_GATE = AUX_Q + 8 * Q_ROW_STRIDE;  // bf16 [4][128]
constexpr int AUX_BYTES = AUX_GATE + 4 * DV * 2;
constexpr uint32_t Q_TX = HEADS * Q_ROW;
constexpr uint32_t EPI_TX = 4 * DV * 2 + 16;        // gate rows + lambda
}  // namespace dc

// Split-kernel configuration: each consumer warp takes 16 keys of a TK-key
// stage; CTAS_PER_SM CTAs share an SM.
template <int TK_, int CW_, int CTAS_>
struct DCfg {
    static constexpr int TK = TK_;                 // keys per stage
    static constexpr int CONSUMER_WARPS = CW_;
    static constexpr int CTAS_PER_SM = CTAS_;
    static constexpr int NCT = CW_ * 32;           // consumer threads
    static constexpr int NUM_THREADS = NCT + 32;   // + the TMA producer warp
    // merge and epilogue: MT threads, COLS output columns each
    static constexpr int MT = NCT < dc::DV ? NCT : dc::DV;
    static constexpr int COLS = dc::DV / MT;
    static constexpr int K_CHUNK = TK * 128;       // one 64-dim swizzled chunk
    static constexpr int K_STAGE = 3 * K_CHUNK;
    static constexpr int V_STAGE = 2 * K_CHUNK;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + dc::STAGES * K_STAGE;
    static constexpr int OFF_AUX = OFF_V + dc::STAGES * V_STAGE;
    static constexpr int OFF_RED = OFF_AUX + dc::STAGES * dc::AUX_BYTES;  // [warps][5 heads][128] fp32
    static constexpr int RED_BYTES = CW_ * dc::HEADS * dc::DV * 4;
    static constexpr int OFF_ML = OFF_RED + RED_BYTES;             // [warps][8 heads] m, l
    static constexpr int OFF_BAR = OFF_ML + 2 * CW_ * 8 * 4;
    static constexpr int OFF_MISC = OFF_BAR + 2 * dc::STAGES * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    static constexpr uint32_t STAGE_TX = K_STAGE + V_STAGE;
    static_assert(TK == 16 * CW_, "one 16-key MMA block per consumer warp");
    static_assert(dc::DV % MT == 0, "columns per merge thread");
    static_assert(TK <= 256, "TMA box height");
    static_assert(SMEM_BYTES * CTAS_ <= 232448, "shared memory per SM");
};
// Several splits (long caches): one item per CTA, 64-key stages, 4 consumer warps.
using SplitCfg = DCfg<64, 4, 2>;
// One split (windows, short caches): few small items per SM, whose latency
// chains dominate; 32-key stages and 2 consumer warps let 4 persistent CTAs
// (4 items in flight) share each SM.
using WindowCfg = DCfg<32, 2, 4>;

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

// Key range of one (split, group, sequence) item; an item is empty when the
// sequence's length is invalid or the split starts past its keys.
struct DecodeItem {
    int b, group, split;
    int start;            // packed cache row of the sequence's first key
    int k_begin, k_end;   // keys of this split, positions within the sequence
    int n_stages;
};

__device__ __forceinline__ int decode_visible_keys_of(int start_, int end, const DecodePlan &plan, int &start,
                                                      int &lo) {
    start = start_;
    const int len = end - start;
    const bool ok = (start >= 0) && (len >= 1) && (len <= plan.max_seqlen_k) && (end <= plan.num_cache_rows);
    lo = (plan.window > 0) ? max(0, len - plan.window) : 0;
    return ok ? len - lo : 0;
}
__device__ __forceinline__ int decode_visible_keys(const int32_t *__restrict__ cu, int b, const DecodePlan &plan,
                                                   int &start, int &lo) {
    return decode_visible_keys_of(cu[b], cu[b + 1], plan, start, lo);
}

// Item w given its sequence's cache bounds cu[b], cu[b+1] (read by the caller).
__device__ __forceinline__ DecodeItem decode_item(int cu_b, int cu_b1, int w, const DecodePlan &plan, int tk) {
    DecodeItem d;
    d.split = w % plan.num_splits;
    const int rest = w / plan.num_splits;
    d.group = rest % plan.hkv;
    d.b = rest / plan.hkv;
    int lo;
    const int n_vis = decode_visible_keys_of(cu_b, cu_b1, plan, d.start, lo);
    d.k_begin = lo + d.split * plan.split_keys;
    d.k_end = lo + min(n_vis, (d.split + 1) * plan.split_keys);
    d.n_stages = max(0, (d.k_end - d.k_begin + tk - 1) / tk);
    return d;
}

// Persistent split kernel: every CTA loops over (split, group, sequence)
// items; the producer's stage ring runs on across items, so the next item's
// keys stream in while the current one is computed. The producer alone reads
// the sequence bounds and the item's queries, gate logits and lambda: it puts
// the item's key range into every stage it issues (an empty item gets one
// stage carrying only that) and copies the rest into the item's first stage.
template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, C::CTAS_PER_SM)
gdla_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __nv_bfloat16 *__restrict__ q_sig, const __nv_bfloat16 *__restrict__ q_noise,
                         const int32_t *__restrict__ cu_seqlens_k, const float *__restrict__ lambda,
                         const __nv_bfloat16 *__restrict__ gate, __nv_bfloat16 *__restrict__ out,
                         float *__restrict__ ws, const DecodePlan plan) {
    using namespace dc;
    constexpr int TK = C::TK, CONSUMER_WARPS = C::CONSUMER_WARPS, NCT = C::NCT, MT = C::MT, COLS = C::COLS;
    constexpr int K_CHUNK = C::K_CHUNK, K_STAGE = C::K_STAGE, V_STAGE = C::V_STAGE;
    constexpr int OFF_K = C::OFF_K, OFF_V = C::OFF_V, OFF_AUX = C::OFF_AUX, OFF_RED = C::OFF_RED;
    constexpr int OFF_ML = C::OFF_ML, OFF_BAR = C::OFF_BAR, OFF_MISC = C::OFF_MISC;
    constexpr uint32_t STAGE_TX = C::STAGE_TX;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *empty = full + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC);
    float *red = reinterpret_cast<float *>(smem + OFF_RED);
    float *ml = reinterpret_cast<float *>(smem + OFF_ML);

    const int hkv = plan.hkv;
    const int ns = plan.num_splits;
    const int n_work = ns * hkv * plan.batch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, CONSUMER_WARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Query rows 5..7 of every stage (the unused MMA columns) stay zero; the
    // producer's copies never touch them.
    for (int i = threadIdx.x; i < STAGES * 3 * (Q_ROW_STRIDE / 4); i += C::NUM_THREADS) {
        const int st = i / (3 * (Q_ROW_STRIDE / 4)), r = i % (3 * (Q_ROW_STRIDE / 4));
        reinterpret_cast<uint32_t *>(smem + OFF_AUX + st * AUX_BYTES + AUX_Q + 5 * Q_ROW_STRIDE)[r] = 0u;
    }
    __syncthreads();

    if (warp == CONSUMER_WARPS) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int g = 0, issued = 0;  // stages issued by this CTA (ring position)
            bool ok = true;
            // Sequence bounds one item ahead, so their load latency overlaps the
            // current item's copies.
            const auto seq_of = [&](int ww) { return (ww / ns) / hkv; };
            int nb0 = 0, nb1 = 0;
            if (blockIdx.x < n_work) {
                nb0 = __ldg(cu_seqlens_k + seq_of(blockIdx.x));
                nb1 = __ldg(cu_seqlens_k + seq_of(blockIdx.x) + 1);
            }
            for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
                const int cb0 = nb0, cb1 = nb1;
                const int wn = w + gridDim.x;
                if (wn < n_work) {
                    nb0 = __ldg(cu_seqlens_k + seq_of(wn));
                    nb1 = __ldg(cu_seqlens_k + seq_of(wn) + 1);
                }
                const DecodeItem d = decode_item(cb0, cb1, w, plan, TK);
                const int n_issue = max(1, d.n_stages);
                for (int it = 0; it < n_issue; ++it, ++g) {
                    const int st = g % STAGES;
                    if (g >= STAGES &&
                        !mbar_wait(empty + st, ((g / STAGES) + 1) & 1, abort_flag, ERR_SITE_DECODE | 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *aux = smem + OFF_AUX + st * AUX_BYTES;
                    *reinterpret_cast<int4 *>(aux + AUX_DESC) = make_int4(d.start, d.k_begin, d.k_end, d.n_stages);
                    issued = g + 1;
                    if (d.n_stages == 0) {
                        mbar_arrive(full + st);  // the key range only (release orders the write above)
                        continue;
                    }
                    const bool first = (it == 0);
                    mbar_arrive_expect_tx(full + st, STAGE_TX + (first ? Q_TX + (ns == 1 ? EPI_TX : 0u) : 0u));
                    if (first) {
                        const size_t srow = static_cast<size_t>(d.b) * 4 * hkv + 4 * d.group;  // first signal head
                        for (int i = 0; i < 4; ++i)
                            bulk_load(aux + AUX_Q + i * Q_ROW_STRIDE, q_sig + (srow + i) * DQK, Q_ROW, full + st);
                        bulk_load(aux + AUX_Q + 4 * Q_ROW_STRIDE,
                                  q_noise + (static_cast<size_t>(d.b) * hkv + d.group) * DQK, Q_ROW, full + st);
                        if (ns == 1) {
                            bulk_load(aux + AUX_GATE, gate + srow * DV, 4 * DV * 2, full + st);
                            bulk_load(aux + AUX_LAM, lambda + srow, 16, full + st);
                        }
                    }
                    const int row = d.start + d.k_begin + it * TK;
                    for (int c = 0; c < 3; ++c)
                        tma_load_3d(smem + OFF_K + st * K_STAGE + c * K_CHUNK, &tm_k, full + st, c * 64, d.group, row);
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(smem + OFF_V + st * V_STAGE + c * K_CHUNK, &tm_v, full + st, c * 64, d.group, row);
                }
            }
            if (*abort_flag)
                for (int k = max(0, issued - STAGES); k < issued; ++k)
                    mbar_wait_cycles(full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
        }
    } else {
        // ------------------------------- consumers --------------------------------
        const int g8 = lane >> 2, c = lane & 3;
        const int mi = lane >> 3, ri = lane & 7;
        const int tid = threadIdx.x;     // merge/epilogue: threads < MT own columns tid + j * MT
        const bool merger = tid < MT;
        const float c_log2 = 0.07216878364870322f * 1.4426950408889634f;  // log2(e) / sqrt(192)
        int g = 0;  // stages consumed by this CTA
        bool ok = true;
        for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
            // The item's first stage carries its key range (and its queries).
            int st = g % STAGES;
            if (!__all_sync(0xffffffffu, mbar_wait(full + st, (g / STAGES) & 1, abort_flag, ERR_SITE_DECODE | 2))) {
                ok = false;
                break;
            }
            const uint8_t *aux = smem + OFF_AUX + st * AUX_BYTES;
            const int4 desc = *reinterpret_cast<const int4 *>(aux + AUX_DESC);
            const int k_begin = desc.y, k_end = desc.z, n_stages = desc.w;
            const size_t orow0 = static_cast<size_t>(w / ns) * 4;  // (b * hkv + group) * 4: first signal row
            if (n_stages == 0) {
                // No visible key. Several splits: the combine kernel skips this
                // split. One split: the sequence's output is zero.
                if (ns == 1 && merger) {
#pragma unroll
                    for (int j = 0; j < COLS; ++j)
#pragma unroll
                        for (int i = 0; i < 4; ++i) out[(orow0 + i) * DV + tid + j * MT] = __float2bfloat16_rn(0.f);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + st);
                ++g;
                continue;
            }
            // Q^T fragments (B operand): thread holds head g8, dims 16*ks + 2c(+1) and +8;
            // one ldmatrix.x4 gives two 16-dim steps (rows 5..7 are the zero heads).
            uint32_t qf[DQK / 16][2];
            {
                const uint32_t qb = smem_u32(aux + AUX_Q) + ri * Q_ROW_STRIDE + (mi & 1) * 16 + (mi >> 1) * 32;
#pragma unroll
                for (int ks2 = 0; ks2 < DQK / 32; ++ks2)
                    ldsm_x4(qb + ks2 * 64, qf[2 * ks2][0], qf[2 * ks2][1], qf[2 * ks2 + 1][0], qf[2 * ks2 + 1][1]);
            }
            float lam_pre[4] = {0.f, 0.f, 0.f, 0.f}, g_pre[COLS][4] = {};
            if (ns == 1 && merger) {
                const float *lam_s = reinterpret_cast<const float *>(aux + AUX_LAM);
                const __nv_bfloat16 *gate_s = reinterpret_cast<const __nv_bfloat16 *>(aux + AUX_GATE);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    lam_pre[i] = lam_s[i];
#pragma unroll
                    for (int j = 0; j < COLS; ++j) g_pre[j][i] = __bfloat162float(gate_s[i * DV + tid + j * MT]);
                }
            }
            float o[DV / 16][4];
#pragma unroll
            for (int mt = 0; mt < DV / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
            float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of heads 2c, 2c+1
            float l0 = 0.f, l1 = 0.f;              // this thread's partial sums

            for (int it = 0; it < n_stages; ++it, ++g) {
                st = g % STAGES;
                if (it > 0 &&
                    !__all_sync(0xffffffffu, mbar_wait(full + st, (g / STAGES) & 1, abort_flag, ERR_SITE_DECODE | 2))) {
                    ok = false;
                    break;
                }
                const uint32_t kb = smem_u32(smem + OFF_K + st * K_STAGE);
                const uint32_t vb = smem_u32(smem + OFF_V + st * V_STAGE);
                const int key0 = warp * 16;  // this warp's 16 keys within the stage
                // S^T = K Q^T
                float sacc[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const int krow = key0 + ri + 8 * (mi & 1);
#pragma unroll
                    for (int ks = 0; ks < DQK / 16; ++ks) {
                        const int dim = ks * 16 + 8 * (mi >> 1);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(kb + (dim >> 6) * K_CHUNK + swz(krow, (dim & 63) >> 3), a0, a1, a2, a3);
                        mma_bf16(sacc, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                    }
                }
                // mask keys past the split end (and the cache rows of other sequences)
                const int ubase = k_begin + it * TK + key0;
                if (ubase + g8 >= k_end) { sacc[0] = -INFINITY; sacc[1] = -INFINITY; }
                if (ubase + g8 + 8 >= k_end) { sacc[2] = -INFINITY; sacc[3] = -INFINITY; }
                float mx0 = fmaxf(sacc[0], sacc[2]) * c_log2, mx1 = fmaxf(sacc[1], sacc[3]) * c_log2;
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
                const float p0 = fast_exp2(fmaf(sacc[0], c_log2, -b0));
                const float p1 = fast_exp2(fmaf(sacc[1], c_log2, -b1));
                const float p2 = fast_exp2(fmaf(sacc[2], c_log2, -b0));
                const float p3 = fast_exp2(fmaf(sacc[3], c_log2, -b1));
                l0 = l0 * a0s + p0 + p2;
                l1 = l1 * a1s + p1 + p3;
#pragma unroll
                for (int mt = 0; mt < DV / 16; ++mt) {
                    o[mt][0] *= a0s;
                    o[mt][1] *= a1s;
                    o[mt][2] *= a0s;
                    o[mt][3] *= a1s;
                }
                // P^T blocks (keys g8 / g8+8, heads 2c..2c+1) -> transposed B fragments
                const uint32_t pb0 = movmatrix_t(pack_bf16x2(p0, p1));
                const uint32_t pb1 = movmatrix_t(pack_bf16x2(p2, p3));
                {
                    const int vrow = key0 + ri + 8 * (mi >> 1);
#pragma unroll
                    for (int mt = 0; mt < DV / 16; ++mt) {
                        const int dv = mt * 16 + 8 * (mi & 1);
                        uint32_t v0, v1, v2, v3;
                        ldsm_x4_t(vb + (dv >> 6) * K_CHUNK + swz(vrow, (dv & 63) >> 3), v0, v1, v2, v3);
                        mma_bf16(o[mt], v0, v1, v2, v3, pb0, pb1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + st);
            }
            if (!ok) break;
            // ---- merge the warps: per head max, then rescaled sums ----
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            if (g8 == 0) {
                ml[(warp * 8 + 2 * c) * 2 + 0] = m0;
                ml[(warp * 8 + 2 * c) * 2 + 1] = l0;
                ml[(warp * 8 + 2 * c + 1) * 2 + 0] = m1;
                ml[(warp * 8 + 2 * c + 1) * 2 + 1] = l1;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(NCT) : "memory");
            float gm0 = -INFINITY, gm1 = -INFINITY;
#pragma unroll
            for (int w4 = 0; w4 < CONSUMER_WARPS; ++w4) {
                gm0 = fmaxf(gm0, ml[(w4 * 8 + 2 * c) * 2]);
                gm1 = fmaxf(gm1, ml[(w4 * 8 + 2 * c + 1) * 2]);
            }
            const float f0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - gm0);
            const float f1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - gm1);
            float *rw = red + warp * HEADS * DV;
#pragma unroll
            for (int mt = 0; mt < DV / 16; ++mt) {
                const int dv0 = mt * 16 + g8;
                if (2 * c < HEADS) {
                    rw[(2 * c) * DV + dv0] = o[mt][0] * f0;
                    rw[(2 * c) * DV + dv0 + 8] = o[mt][2] * f0;
                }
                if (2 * c + 1 < HEADS) {
                    rw[(2 * c + 1) * DV + dv0] = o[mt][1] * f1;
                    rw[(2 * c + 1) * DV + dv0 + 8] = o[mt][3] * f1;
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(NCT) : "memory");
            if (merger) {
                // each merge thread sums the warps for every head of its columns, fixed order
                float hm[HEADS], hl[HEADS];
#pragma unroll
                for (int h = 0; h < HEADS; ++h) {
                    float M = -INFINITY;
#pragma unroll
                    for (int w4 = 0; w4 < CONSUMER_WARPS; ++w4) M = fmaxf(M, ml[(w4 * 8 + h) * 2]);
                    float Ls = 0.f;
#pragma unroll
                    for (int w4 = 0; w4 < CONSUMER_WARPS; ++w4) {
                        const float mw = ml[(w4 * 8 + h) * 2];
                        Ls += ml[(w4 * 8 + h) * 2 + 1] * ((mw == -INFINITY) ? 0.f : fast_exp2(mw - M));
                    }
                    hm[h] = M;
                    hl[h] = Ls;
                }
#pragma unroll
                for (int j = 0; j < COLS; ++j) {
                    const int col = tid + j * MT;
                    float hsum[HEADS];
#pragma unroll
                    for (int h = 0; h < HEADS; ++h) {
                        float Os = 0.f;
#pragma unroll
                        for (int w4 = 0; w4 < CONSUMER_WARPS; ++w4) Os += red[(w4 * HEADS + h) * DV + col];
                        hsum[h] = Os;
                    }
                    if (ns == 1) {
                        // one split holds every key: finish here (gate values staged with the item)
                        float hv[HEADS];
#pragma unroll
                        for (int h = 0; h < HEADS; ++h) hv[h] = (hl[h] > 0.f) ? hsum[h] / hl[h] : 0.f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float dd = hv[i] - lam_pre[i] * hv[4];
                            out[(orow0 + i) * DV + col] =
                                __float2bfloat16_rn(__fdividef(dd, 1.f + __expf(-g_pre[j][i])));
                        }
                    } else {
                        const size_t slot = static_cast<size_t>(w);  // ((b * hkv + group) * ns + split)
                        float *wo = ws + slot * (HEADS * DV);
#pragma unroll
                        for (int h = 0; h < HEADS; ++h) wo[h * DV + col] = hsum[h];
                        if (j == 0 && tid < HEADS) {
                            float *wml = ws + plan.ml_offset_floats + slot * (HEADS * 2);
#pragma unroll
                            for (int h = 0; h < HEADS; ++h)
                                if (tid == h) {
                                    wml[h * 2 + 0] = hm[h];
                                    wml[h * 2 + 1] = hl[h];
                                }
                        }
                    }
                }
            }
            // every consumer is done with ml/red before the next item writes them
            asm volatile("bar.sync 1, %0;" ::"n"(NCT) : "memory");
        }
    }
}

// Split merge: one CTA of 5 warps per (sequence, group); warp h merges head h
// over the splits that hold keys of this sequence (the split kernel writes
// nothing for the others). Lanes walk the splits: a shuffle max gives the
// global m, each split gets weight exp2(m_s - m), and each lane then owns 4 dv
// columns of the weighted sum.
__global__ void __launch_bounds__(160)
gdla_decode_combine_kernel(const float *__restrict__ ws, const int32_t *__restrict__ cu_seqlens_k,
                           const float *__restrict__ lambda, const __nv_bfloat16 *__restrict__ gate,
                           __nv_bfloat16 *__restrict__ out, const DecodePlan plan) {
    using namespace dc;
    __shared__ float hbuf[HEADS * DV];
    __shared__ float wsh[HEADS][64];
    const int group = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hkv = plan.hkv;
    const int ns = plan.num_splits;
    int start, lo;
    const int n_vis = decode_visible_keys(cu_seqlens_k, b, plan, start, lo);
    const int ns_b = min(ns, (n_vis + plan.split_keys - 1) / plan.split_keys);  // splits holding keys
    const size_t slot0 = (static_cast<size_t>(b) * hkv + group) * ns;
    const float *wml = ws + plan.ml_offset_floats;
    const int h = warp;
    float M = -INFINITY;
    for (int s = lane; s < ns_b; s += 32) M = fmaxf(M, wml[(slot0 + s) * (HEADS * 2) + h * 2]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float Lsum = 0.f;
    for (int s = lane; s < ns_b; s += 32) {
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
    for (int s = 0; s < ns_b; ++s) {
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

int decode_smem_bytes() { return SplitCfg::SMEM_BYTES; }

int decode_key_tile(const DecodePlan &plan) { return plan.num_splits == 1 ? WindowCfg::TK : SplitCfg::TK; }

template <class C>
static cudaError_t launch_split(const DecodeLaunch &L, const DecodePlan &plan, int dev, int num_sms,
                                cudaStream_t stream) {
    // shared-memory opt-in once per device
    static PerContextFlag attr_set;  // per device, for the context it was set in
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        cudaError_t e = cudaFuncSetAttribute(gdla_decode_split_kernel<C>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    // One split per sequence (windows, short caches): few small items whose
    // latency chains dominate, so persistent CTAs (all resident) pipeline them.
    // Several splits: many items of similar size, balanced best by the hardware
    // scheduler with one item per CTA (the same kernel, one loop trip each).
    const long long work = static_cast<long long>(plan.num_splits) * plan.hkv * plan.batch;
    const long long resident = static_cast<long long>(C::CTAS_PER_SM) * num_sms;
    const unsigned grid = static_cast<unsigned>((plan.num_splits == 1 && work > resident) ? resident : work);
    gdla_decode_split_kernel<C><<<grid, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(
        L.tm_k, L.tm_v, L.q_sig, L.q_noise, L.cu_seqlens_k, L.lambda, L.gate, L.out, L.ws, plan);
    return cudaPeekAtLastError();
}

cudaError_t launch_decode(const DecodeLaunch &L, const DecodePlan &plan, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int num_sms = device_sm_count(dev);
    if (num_sms <= 0) return cudaErrorInvalidDevice;
    // The K/V tensor maps were encoded with decode_key_tile(plan) rows per box.
    e = (plan.num_splits == 1) ? launch_split<WindowCfg>(L, plan, dev, num_sms, stream)
                               : launch_split<SplitCfg>(L, plan, dev, num_sms, stream);
    if (e != cudaSuccess || plan.num_splits == 1) return e;
    dim3 grid2(plan.hkv, plan.batch);
    gdla_decode_combine_kernel<<<grid2, 160, 0, stream>>>(L.ws, L.cu_seqlens_k, L.lambda, L.gate, L.out, plan);
    return cudaPeekAtLastError();
}

}  // namespace gdla
