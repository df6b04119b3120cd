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
// RMSNorm(c) W = rsqrt(mean(c^2) + eps) * ((c * gamma) W): the row scale is one scalar
// per token, so it moves from the up-projections' operand to their epilogue. Two
// launches of one persistent grouped GEMM (weights [out_features, in_features] bf16,
// K-major):
//   phase 1, A = x (K = 4096): gate logits (bf16 [N, 4H, 128]); c^Q (256-column tiles:
//            c^Q * gamma_q in bf16 and the tile's partial sums of squares); [c^KV; k^R]
//            (192-column tiles: c^KV * gamma_kv in bf16 and partial sums of squares; for
//            the k^R columns the rotary table cos/sin(t base^(-i/32)), angles in fp64, and
//            the rotated k^R); lambda (sigmoid, fp32 [N, 4H]);
//   phase 2: (c^Q * gamma_q) W^Q_b (K = 1024, 256-column tiles of the 5H x 192 query
//            columns, scaled by the row's rsqrt, each head's rotary 64 columns rotated)
//            -> q_sig, q_noise; and
//            (c^KV * gamma_kv) W^UK_j, (c^KV * gamma_kv) W^UV_j (K = 512, one KV head per
//            128-column tile, scaled) -> k = [k_nope | rotated k^R], v.
// The GEMM: CTA pairs (clusters of two, one CTA per SM) walk 256-row x nt-column tiles
// (t = pair, + pairs, ...). In each CTA a TMA producer warp streams 64-wide K chunks of
// its 128 rows of A and its half of the tile's B rows (the weights' rows) through a
// 5- or 6-stage ring; one elected thread of the even CTA issues the pair's tcgen05 MMAs
// (cta_group::2, M = 256, N = nt, fp32) into one of two TMEM accumulators, so 8
// epilogue warps per CTA (TMEM lane quarter = warp % 4, column half = warp / 4) drain
// one tile while the next one is multiplied. Each SM loads 128 + nt/2 operand rows
// per K chunk instead of 128 + nt.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdla_internal.h"
#include "gdla_prologue.h"
#include "gdla_pair.cuh"
#include "gdla_ptx.cuh"

namespace gdla {

// Epilogue modes of the projection GEMM.
enum : int { PRO_CQ = 0, PRO_CKV = 1, PRO_LAMBDA = 2, PRO_GATE = 3, PRO_QUP = 4, PRO_KUP = 5, PRO_VUP = 6 };

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
constexpr int A_BYTES = 128 * 128;             // 128 rows x 64 K (bf16)
constexpr int EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8, MMA_WARP = 9;
constexpr int NUM_THREADS = 320;
constexpr uint32_t ACC_COLS = 256;             // column offset of the second accumulator
constexpr uint32_t TMEM_COLS = 512;
constexpr int SSQ = 16;                        // partial sums of squares per row
}  // namespace pg

// Shared memory of a phase: a ring of A chunks and half-B chunks (up to 128 rows; 6
// stages in phase 1, 5 in phase 2); phase 2 adds four 4 KB output boxes (32 rows x 64
// bf16, 128-byte swizzle) per TMEM lane quarter, shared by the quarter's two epilogue
// warps and read by their TMA stores.
template <int PHASE>
struct PhaseCfg {
    static constexpr int STAGES = PHASE == 1 ? 6 : 5;
    static constexpr int B_ROWS = 128;
    static constexpr int STAGE = pg::A_BYTES + B_ROWS * 128;
    static constexpr int OFF_STG = STAGES * STAGE;
    static constexpr int STG_BYTES = PHASE == 1 ? 0 : 4 * 4 * 4096;
    static constexpr int OFF_BAR = OFF_STG + STG_BYTES;  // full[S], empty[S], acc_full[2], acc_empty[2], drain
    static constexpr int OFF_MISC = OFF_BAR + 32 * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(2 * STAGES + 9 <= 32, "barrier slots");
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

struct TileRef {
    int p, n_tile, m0;
};
// Tile t: problem p, column tile n_tile, first row m0 of its 256-row pair block.
__device__ __forceinline__ TileRef decode_tile(const ProjGroup &G, int t) {
    int p = 0;
    while (p + 1 < G.n_prob && t >= G.prob[p + 1].first) ++p;
    const int local = t - G.prob[p].first;
    return {p, local / G.m_pairs, (local % G.m_pairs) * 256};
}

// ------------------------------ phase 1 epilogues -----------------------------
// 32 values c -> bf16 (c * gamma) at dst; returns the sum of squares of the c.
__device__ __forceinline__ float scale_store_32(__nv_bfloat16 *dst, uint32_t (&o)[32], const float *gamma,
                                                bool row_ok) {
    const float4 *g4 = reinterpret_cast<const float4 *>(gamma);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 g = __ldg(g4 + i);
        const float gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x = __uint_as_float(o[4 * i + j]);
            ss = fmaf(x, x, ss);
            o[4 * i + j] = __float_as_uint(x * gv[j]);
        }
    }
    if (row_ok) store_bf16_32(dst, o);
    return ss;
}

// c^Q tile (256 columns): this half's 128 columns.
__device__ __forceinline__ void epi_cq(const PrologueIO &io, uint32_t tcol, int m, bool row_ok, int n_tile,
                                       int hf) {
    const int c0 = n_tile * 256 + hf * 128;
    float ss = 0.f;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld32(tcol + hf * 128 + ch * 32, o);
        ss += scale_store_32(io.cq_g + static_cast<size_t>(m) * 1024 + c0 + ch * 32, o, io.gamma_q + c0 + ch * 32,
                             row_ok);
    }
    if (row_ok) io.ssq[static_cast<size_t>(m) * pg::SSQ + n_tile * 2 + hf] = ss;
}

// [c^KV; k^R] tile (192 columns): this half's 96 columns. Columns 512..575 are k^R:
// the half that holds them (tile 2, half 1) also writes the row's rotary table and
// the rotated k^R.
__device__ __forceinline__ void epi_ckv(const PrologueIO &io, const ProloguePlan &plan, uint32_t tcol, int m,
                                        bool row_ok, int n_tile, int hf, int lane) {
    const int c0 = n_tile * 192 + hf * 96;
    const bool rope_part = (c0 + 96 > 512);
    const int n_norm = rope_part ? 1 : 3;  // 32-column chunks of c^KV
    float ss = 0.f;
#pragma unroll 1
    for (int ch = 0; ch < n_norm; ++ch) {
        uint32_t o[32];
        tmem_ld32(tcol + hf * 96 + ch * 32, o);
        ss += scale_store_32(io.ckv_g + static_cast<size_t>(m) * 512 + c0 + ch * 32, o, io.gamma_kv + c0 + ch * 32,
                             row_ok);
    }
    if (row_ok) io.ssq[static_cast<size_t>(m) * pg::SSQ + 8 + n_tile * 2 + hf] = ss;
    if (!rope_part) return;
    // this lane's inverse frequency base^(-lane/32) in fp64; the lanes share them by shuffle
    const double inv_lane = exp2(-static_cast<double>(lane) * (13.287712379549449 / 32.0));
    uint32_t a[32], b[32];
    tmem_ld32(tcol + hf * 96 + 32, a);  // k^R dims 0..31
    tmem_ld32(tcol + hf * 96 + 64, b);  // k^R dims 32..63
    const double pos = row_ok ? static_cast<double>(row_position(plan, m)) : 0.0;
    float *rot = io.rot + static_cast<size_t>(m) * 64;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const double inv = __shfl_sync(0xffffffffu, inv_lane, i);
        double s, c;
        sincos(pos * inv, &s, &c);
        if (row_ok) {
            rot[i] = static_cast<float>(c);
            rot[32 + i] = static_cast<float>(s);
        }
        const double x0 = __uint_as_float(a[i]), x1 = __uint_as_float(b[i]);
        a[i] = __float_as_uint(static_cast<float>(x0 * c - x1 * s));
        b[i] = __float_as_uint(static_cast<float>(x0 * s + x1 * c));
    }
    if (row_ok) {
        store_bf16_32(io.krope + static_cast<size_t>(m) * 64, a);
        store_bf16_32(io.krope + static_cast<size_t>(m) * 64 + 32, b);
    }
}

// lambda tile (64 columns of 4H): this half's 32 columns, sigmoid.
__device__ __forceinline__ void epi_lambda(const PrologueIO &io, uint32_t tcol, int m, bool row_ok, int n_tile,
                                           int hf) {
    const int n_out = 4 * io.hkv;
    const int c0 = n_tile * 64 + hf * 32;
    if (c0 >= n_out) return;
    uint32_t o[32];
    tmem_ld32(tcol + hf * 32, o);
    if (!row_ok) return;
    float *dst = io.lambda + static_cast<size_t>(m) * n_out + c0;
    float y[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) y[i] = 1.f / (1.f + __expf(-__uint_as_float(o[i])));
    if (c0 + 32 <= n_out) {
        float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
        for (int i = 0; i < 8; ++i) d4[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (c0 + i < n_out) dst[i] = y[i];
    }
}

// gate tile (256 columns of 4H x 128): this half's 128 columns, bf16.
__device__ __forceinline__ void epi_gate(const PrologueIO &io, uint32_t tcol, int m, bool row_ok, int n_tile,
                                         int hf) {
    __nv_bfloat16 *dst = io.gate + static_cast<size_t>(m) * (4 * io.hkv * 128) + n_tile * 256 + hf * 128;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld32(tcol + hf * 128 + ch * 32, o);
        if (row_ok) store_bf16_32(dst + ch * 32, o);
    }
}

// ------------------------------ phase 2 epilogues -----------------------------
__device__ __forceinline__ void scale_32(uint32_t (&o)[32], float r) {
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * r);
}

// 32 fp32 values (as bits) x r -> bf16 into 16-byte chunks c0..c0+3 of this lane's
// 128-byte row of a 128-byte-swizzled output box at shared address `box`.
__device__ __forceinline__ void stage_32(uint32_t box, int lane, int c0, const uint32_t (&o)[32], float r) {
    const uint32_t row = box + lane * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t w[4] = {pack_bf16x2(__uint_as_float(o[8 * i]) * r, __uint_as_float(o[8 * i + 1]) * r),
                               pack_bf16x2(__uint_as_float(o[8 * i + 2]) * r, __uint_as_float(o[8 * i + 3]) * r),
                               pack_bf16x2(__uint_as_float(o[8 * i + 4]) * r, __uint_as_float(o[8 * i + 5]) * r),
                               pack_bf16x2(__uint_as_float(o[8 * i + 6]) * r, __uint_as_float(o[8 * i + 7]) * r)};
        sts128(row + (((c0 + i) ^ (lane & 7)) << 4), w);
    }
}

// Query up-projection tiles are 256 columns of the row [q_sig heads | q_noise heads]
// (192 per head): box b (64 columns) of tile n starts at column 256 n + 64 b, which is
// dims 0, 64 or 128 of one head (a head's rotary dims 128..191 never straddle a box).
__device__ __forceinline__ bool qup_box_rotary(int n_tile, int b) { return (256 * n_tile + 64 * b) % 192 == 128; }

// Row data an up-projection epilogue reads besides the accumulator, loaded before
// the accumulator is waited for: the partial sums of squares and the row's rotary
// cos | sin (a query half holding a rotary box) or rotated k^R (k_nope tiles, half 1).
struct Epi2Row {
    float4 ss0, ss1;
    float4 rot[16];
};
__device__ __forceinline__ void epi2_prefetch(const PrologueIO &io, int m, bool row_ok, int epi, int hf, int n_tile,
                                              Epi2Row &d) {
    const bool qup = epi == PRO_QUP;
    const size_t row = static_cast<size_t>(row_ok ? m : 0);
    const float4 *p = reinterpret_cast<const float4 *>(io.ssq + row * pg::SSQ);
    d.ss0 = __ldg(p + (qup ? 0 : 2));
    d.ss1 = __ldg(p + (qup ? 1 : 3));
    if (qup && (qup_box_rotary(n_tile, 2 * hf) || qup_box_rotary(n_tile, 2 * hf + 1))) {
        const float4 *rot = reinterpret_cast<const float4 *>(io.rot + row * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i) d.rot[i] = __ldg(rot + i);
    } else if (hf == 1 && epi == PRO_KUP) {
        const float4 *kr = reinterpret_cast<const float4 *>(io.krope + row * 64);  // 64 bf16
#pragma unroll
        for (int i = 0; i < 8; ++i) d.rot[i] = __ldg(kr + i);
    }
}
// rsqrt(mean of squares + eps): c^Q from partial sums 0..7, c^KV from 8..13.
__device__ __forceinline__ float epi2_rsqrt(const Epi2Row &d, bool qup, bool row_ok) {
    if (!row_ok) return 0.f;
    const float s = (d.ss0.x + d.ss0.y) + (d.ss0.z + d.ss0.w) + (d.ss1.x + d.ss1.y);
    return qup ? rsqrtf((s + (d.ss1.z + d.ss1.w)) * (1.f / 1024.f) + 1e-6f) : rsqrtf(s * (1.f / 512.f) + 1e-6f);
}

// One 256-column query tile into the quarter's output boxes `stg`: half hf stages boxes
// 2 hf and 2 hf + 1 (those past the last column are skipped); a box holding a head's
// rotary dims is rotated (pairs i, i + 32) with the row's cos | sin.
__device__ __forceinline__ void epi_qup(const Epi2Row &d, float r, uint32_t tcol, bool row_ok, int n_tile, int hf,
                                        int lane, uint32_t stg, int n_cols) {
#pragma unroll 1
    for (int bb = 0; bb < 2; ++bb) {
        const int b = 2 * hf + bb;
        if (256 * n_tile + 64 * b >= n_cols) break;
        uint32_t a[32], c[32];
        tmem_ld32(tcol + 64 * b, a);
        tmem_ld32(tcol + 64 * b + 32, c);
        if (qup_box_rotary(n_tile, b) && row_ok) {
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
                const float4 c4 = d.rot[i4], s4 = d.rot[8 + i4];
                const float cv[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = 4 * i4 + j;
                    const float x0 = __uint_as_float(a[i]), x1 = __uint_as_float(c[i]);
                    a[i] = __float_as_uint(x0 * cv[j] - x1 * sv[j]);
                    c[i] = __float_as_uint(x0 * sv[j] + x1 * cv[j]);
                }
            }
        }
        stage_32(stg + b * 4096, lane, 0, a, r);
        stage_32(stg + b * 4096, lane, 4, c, r);
    }
}

// One KV head j (tile n = j) of k_nope (PRO_KUP) or v (PRO_VUP): half hf stages
// dims 64 hf .. 64 hf + 63 in box hf; half 1 of k_nope also stages the rotated k^R
// (k's dims 128..191) in box 2.
__device__ __forceinline__ void epi_kvup(const Epi2Row &d, float r, uint32_t tcol, bool is_k, int hf, int lane,
                                         uint32_t stg) {
#pragma unroll 1
    for (int ch = 0; ch < 2; ++ch) {
        uint32_t o[32];
        tmem_ld32(tcol + hf * 64 + ch * 32, o);
        stage_32(stg + hf * 4096, lane, ch * 4, o, r);
    }
    if (!(is_k && hf == 1)) return;
    const uint32_t row = stg + 2 * 4096 + lane * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 v = d.rot[i];
        const uint32_t w[4] = {__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z), __float_as_uint(v.w)};
        sts128(row + ((i ^ (lane & 7)) << 4), w);
    }
}

// ------------------------------------------------------------------------------
// The persistent grouped projection GEMM. PHASE 1 runs PRO_GATE, PRO_CQ, PRO_CKV and
// PRO_LAMBDA problems; PHASE 2 PRO_QUP, PRO_KUP and PRO_VUP.
// ------------------------------------------------------------------------------
template <int PHASE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pg::NUM_THREADS, 1)
gdla_proj_kernel(const __grid_constant__ ProjGroup G, const __grid_constant__ PrologueIO io,
                 const __grid_constant__ ProloguePlan plan) {
    using namespace pg;
    using C = PhaseCfg<PHASE>;
    constexpr int STAGES = C::STAGES, STAGE = C::STAGE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars;                   // [stage]
    uint64_t *empty = bars + STAGES;         // [stage]
    uint64_t *acc_full = bars + 2 * STAGES;  // [accumulator]
    uint64_t *acc_empty = acc_full + 2;      // [accumulator]
    uint64_t *drain = acc_empty + 2;
    uint64_t *qfree = drain + 1;            // [lane quarter] (phase 2): its output boxes are free
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full + i, 1);
            mbar_init(acc_empty + i, 2 * EPI_WARPS);  // both CTAs' epilogue warps (the even CTA's copy)
        }
        mbar_init(drain, 1);
        for (int i = 0; i < 4; ++i) mbar_init(qfree + i, 2);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            uint32_t g = 0, issued = 0;
            bool ok = true;
            for (int t = pair; ok && t < G.total_tiles; t += n_pairs) {
                const TileRef tr = decode_tile(G, t);
                const ProjProblem &pr = G.prob[tr.p];
                const int half = pr.nt >> 1;
                const uint32_t bytes = 2 * (A_BYTES + half * 128);  // both CTAs' loads
                for (int kc = 0; kc < pr.nk; ++kc, ++g) {
                    const uint32_t st = g % STAGES;
                    if (g >= STAGES &&
                        !mbar_wait_cl(empty + st, ((g / STAGES) + 1) & 1, abort_flag, ERR_SITE_PROLOGUE | 1)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(full + st, bytes);
                    uint8_t *sb = smem + st * STAGE;
                    tma_load_3d_pair(sb, &G.tm_a[tr.p], full + st, kc * 64, tr.m0 + 128 * rank, 0);
                    tma_load_3d_pair(sb + A_BYTES, &G.tm_b[tr.p], full + st, kc * 64,
                                     tr.n_tile * pr.nt + half * rank, 0);
                    issued = g + 1;
                }
            }
            if (*abort_flag && even)
                for (uint32_t k = issued > STAGES ? issued - STAGES : 0; k < issued; ++k)
                    mbar_wait_cl_cycles(full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
        }
    } else if (warp == MMA_WARP) {
        if (even) {  // the pair's MMAs are issued by the even CTA
        const uint32_t leader = elect_one_sync();
        const uint64_t a_desc0 = desc_sw128(smem_u32(smem), 16, 1024);
        const uint64_t b_desc0 = desc_sw128(smem_u32(smem + A_BYTES), 16, 1024);
        uint32_t g = 0;
        bool ok = true;
        int i = 0;
        for (int t = pair; ok && t < G.total_tiles; t += n_pairs, ++i) {
            const TileRef tr = decode_tile(G, t);
            const ProjProblem &pr = G.prob[tr.p];
            const int buf = i & 1, use = i >> 1;
            if (use > 0 && !__all_sync(0xffffffffu, mbar_wait_cl(acc_empty + buf, (use - 1) & 1, abort_flag,
                                                                  ERR_SITE_PROLOGUE | 2))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(256, pr.nt, false, false);
            const uint32_t d = tmem + buf * ACC_COLS;
            for (int kc = 0; kc < pr.nk; ++kc, ++g) {
                const uint32_t st = g % STAGES;
                if (!__all_sync(0xffffffffu,
                                mbar_wait_cl(full + st, (g / STAGES) & 1, abort_flag, ERR_SITE_PROLOGUE | 3))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sb = st * STAGE;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ss_pair_leader(d, a_desc0 + ((sb + kk * 32) >> 4), b_desc0 + ((sb + kk * 32) >> 4), idesc,
                                        (kc > 0 || kk > 0) ? 1u : 0u, leader);
                umma_commit_pair_leader(empty + st, leader);
            }
            if (ok) umma_commit_pair_leader(acc_full + buf, leader);
        }
        // every MMA this warp issued has finished before the TMEM is released
        umma_commit_pair_leader(drain, leader);
        mbar_wait_cl_cycles(drain, 0, 1ll << 22);
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int q = warp & 3, hf = warp >> 2;
        const uint32_t stg = smem_u32(smem + C::OFF_STG + q * 4 * 4096);  // the quarter's output boxes
        const uint32_t acc_empty_even = mapa_shared(smem_u32(acc_empty), 0);
        int i = 0;
        for (int t = pair; t < G.total_tiles; t += n_pairs, ++i) {
            TileRef tr = decode_tile(G, t);
            tr.m0 += 128 * rank;  // this CTA's rows of the pair block
            const int buf = i & 1, use = i >> 1;
            const int m = tr.m0 + q * 32 + lane;
            const bool row_ok = m < G.M;
            const int epi = G.prob[tr.p].epi;
            Epi2Row pre;
            if constexpr (PHASE == 2) epi2_prefetch(io, m, row_ok, epi, hf, tr.n_tile, pre);
            if (!__all_sync(0xffffffffu,
                            mbar_wait_cl(acc_full + buf, use & 1, abort_flag, ERR_SITE_PROLOGUE | 4)))
                break;
            tc_fence_after();
            const uint32_t tcol = tmem + buf * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16);
            if constexpr (PHASE == 1) {
                if (epi == PRO_CQ) epi_cq(io, tcol, m, row_ok, tr.n_tile, hf);
                else if (epi == PRO_CKV) epi_ckv(io, plan, tcol, m, row_ok, tr.n_tile, hf, lane);
                else if (epi == PRO_LAMBDA) epi_lambda(io, tcol, m, row_ok, tr.n_tile, hf);
                else epi_gate(io, tcol, m, row_ok, tr.n_tile, hf);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty_even + buf * 8);
            } else {
                // the quarter's boxes are free once both its warps' previous stores have read them
                if (lane == 0) {
                    bulk_wait_group_read0();
                    mbar_arrive(qfree + q);
                }
                if (!__all_sync(0xffffffffu, mbar_wait(qfree + q, i & 1, abort_flag, ERR_SITE_PROLOGUE | 5)))
                    break;
                const bool qup = epi == PRO_QUP;
                const float r = epi2_rsqrt(pre, qup, row_ok);
                const int n_cols = 5 * io.hkv * 192;  // query up-projection columns
                if (qup) epi_qup(pre, r, tcol, row_ok, tr.n_tile, hf, lane, stg, n_cols);
                else epi_kvup(pre, r, tcol, epi == PRO_KUP, hf, lane, stg);
                tc_fence_before();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_cluster(acc_empty_even + buf * 8);
                    const int row0 = tr.m0 + q * 32;
                    if (row0 < G.M) {  // rows past the last token are clipped by the store
                        const int hq = 4 * io.hkv;
                        if (qup) {  // boxes 2 hf, 2 hf + 1: columns 256 n + 64 b = head, dims
                            for (int b = 2 * hf; b < 2 * hf + 2; ++b) {
                                const int col = 256 * tr.n_tile + 64 * b;
                                if (col >= n_cols) break;
                                const int head = col / 192;
                                tma_store_3d(head < hq ? &G.tm_o[0] : &G.tm_o[1],
                                             smem + C::OFF_STG + (q * 4 + b) * 4096, col % 192,
                                             head < hq ? head : head - hq, row0);
                            }
                        } else {  // k / v half hf -> box hf (dims 64 hf ..), k's half 1 also box 2 (k^R)
                            const CUtensorMap *map = epi == PRO_KUP ? &G.tm_o[2] : &G.tm_o[3];
                            const int b_hi = (epi == PRO_KUP && hf) ? 2 : hf;
                            for (int b = hf; b <= b_hi; ++b)
                                tma_store_3d(map, smem + C::OFF_STG + (q * 4 + b) * 4096, 64 * b, tr.n_tile, row0);
                        }
                        bulk_commit_group();
                    }
                }
            }
        }
        if (PHASE == 2 && lane == 0) bulk_wait_group0();
    }
    tc_fence_before();
    cluster_sync();  // no CTA leaves while the pair's MMAs or the peer may still touch it
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------
// The tile's nt B rows are rows n_tile nt .. of b; each CTA of a pair loads one half.
static void add_problem(ProjGroup &G, const CUtensorMap &a, const CUtensorMap &b, int epi, int nt, int K,
                        int n_tiles) {
    const int p = G.n_prob++;
    G.tm_a[p] = a;
    G.tm_b[p] = b;
    G.prob[p] = ProjProblem{epi, nt, K / 64, n_tiles, G.total_tiles};
    G.total_tiles += n_tiles * G.m_pairs;
}

template <int PHASE>
static cudaError_t launch_group(const ProjGroup &G, const PrologueIO &io, const ProloguePlan &plan,
                                cudaStream_t stream) {
    static PerContextFlag attr_set;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        e = cudaFuncSetAttribute(gdla_proj_kernel<PHASE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PhaseCfg<PHASE>::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    // as many pairs as can be resident at once (a cluster's two CTAs need two SMs of
    // one GPC, so this can be below half the SM count)
    static std::atomic<int> max_clusters[kMaxCachedDevices];
    static PerContextFlag clusters_known;
    int nc = 0;
    if (dev >= 0 && dev < kMaxCachedDevices && clusters_known.is_set(dev, ctx)) {
        nc = max_clusters[dev].load(std::memory_order_relaxed);
    } else {
        int sms = device_sm_count(dev);
        if (sms <= 0) sms = 148;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1));
        cfg.blockDim = dim3(pg::NUM_THREADS);
        cfg.dynamicSmemBytes = PhaseCfg<PHASE>::SMEM_BYTES;
        e = cudaOccupancyMaxActiveClusters(&nc, gdla_proj_kernel<PHASE>, &cfg);
        if (e != cudaSuccess) return e;
        if (nc <= 0) return cudaErrorInvalidConfiguration;
        nc = nc < sms / 2 ? nc : sms / 2;
        if (dev >= 0 && dev < kMaxCachedDevices) {
            max_clusters[dev].store(nc, std::memory_order_relaxed);
            clusters_known.set(dev, ctx);
        }
    }
    const int pairs = G.total_tiles < nc ? G.total_tiles : nc;
    gdla_proj_kernel<PHASE><<<2 * pairs, pg::NUM_THREADS, PhaseCfg<PHASE>::SMEM_BYTES, stream>>>(G, io, plan);
    return cudaPeekAtLastError();
}

cudaError_t launch_prologue(const PrologueLaunch &L, const ProloguePlan &plan, int M, cudaStream_t stream) {
    const int hkv = L.io.hkv;
    const int m_pairs = (M + 255) / 256;
    // phase 1: the projections of x, widest tiles first (the tail gets the narrow ones)
    ProjGroup g1{};
    g1.m_pairs = m_pairs;
    g1.M = M;
    add_problem(g1, L.tm_x, L.tm_wgate, PRO_GATE, 256, 4096, 2 * hkv);
    add_problem(g1, L.tm_x, L.tm_wqa, PRO_CQ, 256, 4096, 4);
    add_problem(g1, L.tm_x, L.tm_wkva, PRO_CKV, 192, 4096, 3);
    add_problem(g1, L.tm_x, L.tm_wlam, PRO_LAMBDA, 64, 4096, (4 * hkv + 63) / 64);
    cudaError_t e = launch_group<1>(g1, L.io, plan, stream);
    if (e != cudaSuccess) return e;
    // phase 2: the up-projections
    ProjGroup g2{};
    g2.m_pairs = m_pairs;
    g2.M = M;
    g2.tm_o[0] = L.tm_qs_o;
    g2.tm_o[1] = L.tm_qn_o;
    g2.tm_o[2] = L.tm_k_o;
    g2.tm_o[3] = L.tm_v_o;
    add_problem(g2, L.tm_cqn, L.tm_wqb, PRO_QUP, 256, 1024, (5 * hkv * 192 + 255) / 256);
    add_problem(g2, L.tm_ckvn, L.tm_wuk, PRO_KUP, 128, 512, hkv);
    add_problem(g2, L.tm_ckvn, L.tm_wuv, PRO_VUP, 128, 512, hkv);
    return launch_group<2>(g2, L.io, plan, stream);
}

}  // namespace gdla
