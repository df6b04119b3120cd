// gdla_prefill.cu - packed varlen GDLA prefill for sm_100a.
//
// Method (aitrends.kr/articles/94908, GDLA paragraphs): for each KV head j the
// 4 signal heads 4j..4j+3 and the noise head j run causal softmax attention
// over the same K_j (192) and V_j (128); then D_i = H_S,i - lambda_i * H_N,j
// and out_i = sigmoid(gate_i) * D_i.
//
// Work. A work item is (KV group, block of TILES x 24 consecutive tokens of
// one sequence). CTAs are persistent (one per SM) and take items from a list
// sorted heaviest first, round-robin with the direction reversed every round.
//
// Tiling. In each 24-token tile the 5 query heads fill the M = 128 rows of one
// tensor-core MMA, laid out per TMEM lane quarter (one warp) so that every
// warp owns whole tokens:
//     quarter w (rows 32w..32w+31) holds tokens 6w..6w+5 of the tile:
//       rows 32w + 4*i + h   signal head h (0..3) of token 6w+i   (24 rows)
//       rows 32w + 24 + i    the noise head of token 6w+i         (6 rows)
//       rows 32w + 30, 31    unused (zero queries)
// Each BN-key K/V tile is staged once in shared memory (TMA) and consumed by
// every tile and all five heads. Per key tile k and q tile x:
//     S_x = Q_x K^T   tcgen05 M=128 N=BN K=192, fp32 in TMEM; K from shared
//                     memory, Q from TMEM (one q tile, copied there per item) or
//                     from shared memory (two q tiles)
//     softmax_x       one warpgroup per tile, one TMEM lane per row: online
//                     max/sum, P = exp2(.) rounded to bf16 into TMEM over S_x
//     O_x += P_x V    tcgen05 with A = P from TMEM, B = V from smem (MN-major)
// S is double-buffered per tile, so QK^T of key tile k+1 is queued while the
// softmax of tile k runs; with two q tiles the softmax warpgroups alternate
// (ping-pong). Epilogue: every warp finalises its rows (O/l), passes each
// token's noise row to its four signal rows with warp shuffles, and writes
// sigmoid(g)(H_S - lambda H_N) as bf16 (32-byte gate loads and output stores
// when the buffers allow). Meanwhile the tensor core already
// computes QK^T of the next item (its Q was loaded as soon as the last QK^T
// of the current item finished).
//
// Two configurations (measured on B200: an M=128 MMA from shared memory takes
// the same ~65 cycles at N=64 as at N=128, so 128-key tiles double the tensor
// rate of QK^T):
//   Causal  (TILES=1, BN=128, 2 K + 2 V stages) for full-causal and long windows;
//   Sliding (TILES=2, BN=64, 3 K + 3 V stages) for short windows, where the path
//           is bound by HBM and 48-token items halve the per-token overheads.
// Warps: 4 per q tile (softmax + epilogue), then the TMA producer warp (which
// also zero-fills the unused Q rows once) and the MMA warp (TMEM allocation,
// MMA issue by one elected lane of a converged warp). The plan of a launch (its
// items) travels in the kernel parameters, in one of three capacities.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cstring>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

// One full 32-byte sector per lane (sm_100 256-bit loads/stores); the address
// must be 32-byte aligned.
__device__ __forceinline__ void ld_nc_v8(const void *p, uint32_t *r) {
    asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}
__device__ __forceinline__ void st_v8(void *p, const uint32_t *r) {
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

namespace pf {
constexpr int TOK = kPrefillTileTokens;  // 24 tokens per MMA tile
constexpr int ROWS = 128;
constexpr int SIG_ROWS = 4 * TOK;     // 96
constexpr int NOISE_ROW0 = SIG_ROWS;  // 96
constexpr int DQK = 192, DV = 128;
constexpr int KCHUNKS = DQK / 64;
constexpr int VCHUNKS = DV / 64;
constexpr int Q_CHUNK = ROWS * 128;        // 16 KB
constexpr int Q_TILE = KCHUNKS * Q_CHUNK;  // 48 KB
constexpr uint32_t Q_TX = KCHUNKS * (64 * 4 * TOK * 2 + 64 * 1 * TOK * 2);
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
constexpr int kPolyEvery = 4;              // one exponential pair in 4 on the FMA pipe

// Gate / output staging of the asynchronous epilogue, per q tile: the gate
// logits of its 24 tokens x 4 signal heads as two 128-byte-swizzled boxes
// (dims 0..63, 64..127) of [token][head][64] bf16, 12 KB each; the output is
// written over them in place and stored from there by TMA, one 3 KB box
// (6 tokens) per warp and half.
constexpr int G_HALF = TOK * 4 * 128;      // 12 KB
constexpr int G_TILE = 2 * G_HALF;         // 24 KB
constexpr int G_WARP_BOX = 6 * 4 * 128;    // 3 KB: one warp's tokens in one half
constexpr int LAM_TILE = TOK * 4 * 4;      // 384 B: [token][head] fp32

// Epilogue forms.
enum : int {
    EPI_DIRECT = 0,   // gate rows and lambda loaded by the epilogue, output stored directly
    EPI_STAGED = 1,   // gate and lambda arrive in shared memory by TMA during the item; the
                      // output is written over the gate and leaves by TMA store
    EPI_HALF = 2,     // gate dims 0..63 and lambda staged by TMA during the item (all the
                      // shared memory left), dims 64..127 loaded by the epilogue; output
                      // stored directly
    EPI_BWD = 3,      // backward recompute: instead of the output, the gradients of the
                      // gate, lambda and H (from dout) and the row statistics
};

template <int TILES_, int BN_, int STAGES_, int EPI_>
struct Cfg {
    static constexpr int TILES = TILES_;
    static constexpr int BN = BN_;          // keys per KV tile
    static constexpr int STAGES = STAGES_;
    static constexpr int V_BOX = BN;        // keys per V TMA box
    static constexpr int EPI = EPI_;
    static constexpr bool ASYNC_EPI = EPI == EPI_STAGED || EPI == EPI_HALF;  // gate / lambda staged by the producer
    static constexpr int G_HALVES = EPI == EPI_STAGED ? 2 : (EPI == EPI_HALF ? 1 : 0);
    static constexpr uint32_t GATE_TX = G_HALVES * G_HALF + LAM_TILE;
    static constexpr int CTA_TOK = TILES * TOK;
    static constexpr int KV_CHUNK = BN * 128;            // one 64-dim swizzled chunk
    static constexpr int K_STAGE = KCHUNKS * KV_CHUNK;
    static constexpr int V_STAGE = VCHUNKS * KV_CHUNK;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILES * Q_TILE;
    static constexpr int OFF_V = OFF_K + STAGES * K_STAGE;
    static constexpr int OFF_G = OFF_V + STAGES * V_STAGE;  // 1024-byte aligned (swizzled boxes)
    static constexpr int OFF_LAM = OFF_G + TILES * G_HALVES * G_HALF;
    static constexpr int OFF_BAR = OFF_LAM + (ASYNC_EPI ? TILES * LAM_TILE : 0);
    static constexpr int NUM_BARS = 32;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
    static constexpr uint32_t K_TX = K_STAGE;
    static constexpr uint32_t V_TX = V_STAGE;
    static constexpr uint32_t O_COL0 = 0;              // + 128 * tile
    static constexpr uint32_t S_COL0 = 128 * TILES;    // + 2 * BN * tile + BN * buffer
    // With one q tile, Q is copied into TMEM once per item (96 columns) and
    // QK^T reads it from there, which removes the Q re-reads from shared
    // memory that otherwise bound the MMAs; the shared Q buffer is then only
    // a staging area, free again as soon as the copy is done.
    static constexpr bool Q_IN_TMEM = (TILES == 1);
    static constexpr uint32_t QT_COL0 = S_COL0 + 2 * BN * TILES;
    static constexpr int NUM_THREADS = 128 * TILES + 64;
    static constexpr int PRODUCER_WARP = 4 * TILES;
    static constexpr int MMA_WARP = 4 * TILES + 1;
    static_assert(QT_COL0 + (Q_IN_TMEM ? DQK / 2 : 0) <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(BN == 64 || BN == 128, "key tile");
    static_assert(STAGES <= 3, "three barriers each for K and V stages");
};
using CausalCfg = Cfg<1, 128, 2, EPI_HALF>;
using BwdRecomputeCfg = Cfg<1, 128, 2, EPI_BWD>;         // full causal and long windows: the one-tile schedule
using BwdRecomputeSlidingCfg = Cfg<2, 64, 2, EPI_BWD>;  // short windows: the forward's sliding schedule
using SlidingCfg = Cfg<2, 64, 2, EPI_STAGED>;

// ------------------------------- epilogue ----------------------------------
// Per warp: the 24 signal rows of its 6 tokens. gate/out rows are 256 bytes;
// with 32-byte aligned bases each lane moves whole 32-byte sectors (half the
// memory instructions of 16-byte accesses over the same scattered rows).
// The gated output of 32 columns of this lane's O row, as 16 bf16 pairs:
// H = O/l; the token's noise row H_N comes from lane hsrc by shuffle;
// out = sigmoid(g) (H_S - lambda H_N), in packed fp32 pairs.
__device__ __forceinline__ void epi_gate_pairs(const uint32_t (&o)[32], float inv_l, float lam,
                                               const uint32_t (&g)[16], int hsrc, uint32_t (&res)[16]) {
    const uint64_t inv_l2 = f2_pack(inv_l, inv_l);
    const uint64_t neg_lam2 = f2_pack(-lam, -lam);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint64_t h = f2_mul(f2_pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), inv_l2);
        float h0, h1;
        f2_unpack(h, h0, h1);
        const float n0 = __shfl_sync(0xffffffffu, h0, hsrc);  // H_N of this row's token
        const float n1 = __shfl_sync(0xffffffffu, h1, hsrc);
        const uint64_t d = f2_fma(f2_pack(n0, n1), neg_lam2, h);
        float r0, r1;
        f2_unpack(f2_mul(d, sigmoid2_bf16(g[i])), r0, r1);
        res[i] = pack_bf16x2(r0, r1);
    }
}
// Gate columns 32ch..32ch+31 of one row (16 words of bf16 pairs).
__device__ __forceinline__ void epi_fetch_gate(bool valid, size_t row, const __nv_bfloat16 *__restrict__ gate,
                                               bool wide, int ch, uint32_t (&g)[16]) {
    if (valid) {
        const __nv_bfloat16 *src = gate + row * DV + ch * 32;
        if (wide) {
            ld_nc_v8(src, g);
            ld_nc_v8(src + 16, g + 8);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + i);
                g[4 * i] = v.x;
                g[4 * i + 1] = v.y;
                g[4 * i + 2] = v.z;
                g[4 * i + 3] = v.w;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) g[i] = 0;
    }
}
// Columns 32ch..32ch+31 of this lane's O row: H = O/l; the token's noise row
// comes from lane hsrc by shuffle; out = sigmoid(g) (H_S - lambda H_N) in bf16.
__device__ __forceinline__ void epi_chunk(const uint32_t (&o)[32], float inv_l, float lam, const uint32_t (&g)[16],
                                          int hsrc, bool valid, bool wide, __nv_bfloat16 *__restrict__ dst) {
    uint32_t res[16];
    epi_gate_pairs(o, inv_l, lam, g, hsrc, res);
    if (valid) {
        if (wide) {
            st_v8(dst, res);
            st_v8(dst + 16, res + 8);
        } else {
            uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int i = 0; i < 4; ++i) d[i] = make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]);
        }
    }
}
// This lane's staged gate columns 32ch..32ch+31 (ch 0 or 1 of a 64-dim half):
// 16 words from its 128-byte swizzled row (`key` = row & 7).
__device__ __forceinline__ void epi_gate_staged(bool sig, uint32_t row_addr, int key, int ch, uint32_t (&g)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (sig) {
            lds128(row_addr + ((((ch & 1) * 4 + i) ^ key) << 4), g + 4 * i);
        } else {
            g[4 * i] = g[4 * i + 1] = g[4 * i + 2] = g[4 * i + 3] = 0u;
        }
    }
}
// Asynchronous-epilogue form of epi_chunk: this lane's gate columns
// 32ch..32ch+31 come from its 128-byte row of the swizzled staging box
// (`row_addr` = the row's shared address, `key` = row & 7 selects the
// swizzle); the bf16 result goes back over them (to_smem) or, for a warp
// whose tokens are not all inside the sequence, straight to `dst` (to_global).
__device__ __forceinline__ void epi_chunk_staged(const uint32_t (&o)[32], float inv_l, float lam, int hsrc, bool sig,
                                                 uint32_t row_addr, int key, int ch, bool to_smem, bool to_global,
                                                 __nv_bfloat16 *__restrict__ dst) {
    uint32_t g[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (sig) {
            lds128(row_addr + ((((ch & 1) * 4 + i) ^ key) << 4), g + 4 * i);
        } else {
            g[4 * i] = g[4 * i + 1] = g[4 * i + 2] = g[4 * i + 3] = 0u;
        }
    }
    uint32_t res[16];
    epi_gate_pairs(o, inv_l, lam, g, hsrc, res);
    if (sig && to_smem) {
#pragma unroll
        for (int i = 0; i < 4; ++i) sts128(row_addr + ((((ch & 1) * 4 + i) ^ key) << 4), res + 4 * i);
    }
    if (to_global) {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i) d[i] = make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]);
    }
}

// Backward recompute epilogue (per warp, one TMEM lane = one row): from this
// lane's O row, l and m, the upstream gradient dout and the gate logits,
//   sigma = sigmoid(g), D = H_S - lambda H_N,
//   dgate = dout D sigma (1 - sigma),  dD = dout sigma,  dlambda = -sum dD H_N,
//   dH_S = dD,  dH_N = -sum over the token's 4 signal heads of lambda dD,
// with dH rounded to bf16 (the operand the gradient kernels multiply) and the
// row statistics lse2 = m + log2(l) (so P = exp2(s log2(e)/sqrt(192) - lse2))
// and rowsum(dH * H) taken with that rounded dH.
__device__ __forceinline__ void epi_backward(uint32_t o_addr, float l_run, float m_run, bool is_sig, bool tok_valid,
                                             int lane, int hsrc, size_t tok, int hs, int hkv, int group,
                                             const float *__restrict__ lambda, const __nv_bfloat16 *__restrict__ gate,
                                             const BwdIO &bwd) {
    const bool sig = is_sig && tok_valid;
    const bool noi = lane >= 24 && lane < 30 && tok_valid;
    const size_t srow = tok * hs + 4 * group + (lane & 3);
    const size_t nrow = tok * hkv + group;
    const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
    const float lam = sig ? __ldg(lambda + srow) : 0.f;
    const int nsrc = ((lane - 24) * 4) & 31;  // noise lane 24+i: the first signal lane of token i
    float dl = 0.f, drow = 0.f;
#pragma unroll 1
    for (int ch = 0; ch < DV / 32; ++ch) {
        uint32_t o[32], g[16], go[16];
        tmem_ld32(o_addr + ch * 32, o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 a = make_uint4(0, 0, 0, 0), c = a;
            if (sig) {
                a = __ldg(reinterpret_cast<const uint4 *>(gate + srow * DV + ch * 32) + i);
                c = __ldg(reinterpret_cast<const uint4 *>(bwd.dout + srow * DV + ch * 32) + i);
            }
            g[4 * i] = a.x, g[4 * i + 1] = a.y, g[4 * i + 2] = a.z, g[4 * i + 3] = a.w;
            go[4 * i] = c.x, go[4 * i + 1] = c.y, go[4 * i + 2] = c.z, go[4 * i + 3] = c.w;
        }
        uint32_t w_dgate[16], w_dh[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float h0 = __uint_as_float(o[2 * i]) * inv_l, h1 = __uint_as_float(o[2 * i + 1]) * inv_l;
            const float hn0 = __shfl_sync(0xffffffffu, h0, hsrc), hn1 = __shfl_sync(0xffffffffu, h1, hsrc);
            const float o0 = __uint_as_float(go[i] << 16), o1 = __uint_as_float(go[i] & 0xFFFF0000u);
            float s0, s1;  // sigmoid of the gate pair, one tanh for both
            f2_unpack(sigmoid2_bf16(g[i]), s0, s1);
            const float d0 = h0 - lam * hn0, d1 = h1 - lam * hn1;
            const float dD0 = o0 * s0, dD1 = o1 * s1;
            w_dgate[i] = pack_bf16x2(o0 * d0 * s0 * (1.f - s0), o1 * d1 * s1 * (1.f - s1));
            dl -= dD0 * hn0 + dD1 * hn1;
            // dH_N: the token's 4 signal lanes (4i..4i+3) sum -lambda dD; noise lane 24+i takes it
            float c0 = -lam * dD0, c1 = -lam * dD1;
            c0 += __shfl_xor_sync(0xffffffffu, c0, 1);
            c1 += __shfl_xor_sync(0xffffffffu, c1, 1);
            c0 += __shfl_xor_sync(0xffffffffu, c0, 2);
            c1 += __shfl_xor_sync(0xffffffffu, c1, 2);
            const float n0 = __shfl_sync(0xffffffffu, c0, nsrc), n1 = __shfl_sync(0xffffffffu, c1, nsrc);
            const uint32_t dh = is_sig ? pack_bf16x2(dD0, dD1) : pack_bf16x2(n0, n1);
            w_dh[i] = dh;
            drow += __uint_as_float(dh << 16) * h0 + __uint_as_float(dh & 0xFFFF0000u) * h1;
        }
        if (sig) {
            uint4 *dg = reinterpret_cast<uint4 *>(bwd.dgate + srow * DV + ch * 32);
            uint4 *dh = reinterpret_cast<uint4 *>(bwd.dh_sig + srow * DV + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dg[i] = make_uint4(w_dgate[4 * i], w_dgate[4 * i + 1], w_dgate[4 * i + 2], w_dgate[4 * i + 3]);
                dh[i] = make_uint4(w_dh[4 * i], w_dh[4 * i + 1], w_dh[4 * i + 2], w_dh[4 * i + 3]);
            }
        } else if (noi) {
            uint4 *dh = reinterpret_cast<uint4 *>(bwd.dh_noise + nrow * DV + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dh[i] = make_uint4(w_dh[4 * i], w_dh[4 * i + 1], w_dh[4 * i + 2], w_dh[4 * i + 3]);
        }
    }
    if (sig) bwd.dlambda[srow] = dl;
    if (sig || noi) {
        float *st = bwd.stats + nrow * kBwdStats + (sig ? (lane & 3) : 4);
        st[0] = m_run + log2f(l_run);
        st[8] = drow;
    }
}

}  // namespace pf

template <class C, class Plan>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
gdla_prefill_kernel(const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_qn,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_gate, const __grid_constant__ CUtensorMap tm_lam,
                    const __grid_constant__ CUtensorMap tm_out, const float *__restrict__ lambda,
                    const __nv_bfloat16 *__restrict__ gate, __nv_bfloat16 *__restrict__ out, const BwdIO bwd,
                    const __grid_constant__ Plan plan) {
    using namespace pf;
    constexpr int TILES = C::TILES, BN = C::BN, STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars + 0;    // [tile]: one phase per item
    uint64_t *q_empty = bars + 2;   // [tile]: one phase per item, after its last QK^T
    uint64_t *k_full = bars + 4;    // [stage]
    uint64_t *k_empty = bars + 7;   // [stage]
    uint64_t *v_full = bars + 10;   // [stage]
    uint64_t *v_empty = bars + 13;  // [stage]
    uint64_t *s_full = bars + 16;   // [tile * 2 + buffer]
    uint64_t *p_full = bars + 20;   // [tile * 2 + buffer]
    uint64_t *o_done = bars + 24;   // [tile]: one phase per PV product of the tile
    uint64_t *o_final = bars + 26;  // [tile]: one phase per item, its last PV product is done
    uint64_t *g_full = bars + 28;   // [tile]: one phase per item, its gate and lambda landed (async epilogue)
    uint64_t *g_empty = bars + 30;  // [tile]: one phase per item, its output left the staging buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int hkv = plan.hkv;
    const int hs = 4 * hkv;
    const int window = plan.window;
    const int n_work = plan.n_items * hkv;

    // Item w: group = w % hkv, block = items[w / hkv]; key tiles of q tile x.
    struct Item {
        int group, s0, L, t0, kv_lo;
        int n_tiles[TILES];
    };
    auto item_at = [&](int w) {
        Item it;
        it.group = w % hkv;
        const uint32_t code = plan.items[w / hkv];
        const int seq = static_cast<int>(code >> kItemSeqShift);
        it.s0 = plan.seq_start[seq];
        it.L = plan.seq_len[seq];
        it.t0 = static_cast<int>(code & kItemTileMask) * C::CTA_TOK;
        it.kv_lo = (window > 0) ? max(0, it.t0 - window + 1) : 0;
#pragma unroll
        for (int x = 0; x < TILES; ++x)
            it.n_tiles[x] = (min(it.L, it.t0 + (x + 1) * TOK) - it.kv_lo + BN - 1) / BN;
        return it;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < TILES; ++i) {
            mbar_init(q_full + i, 1);
            mbar_init(q_empty + i, 1);
            mbar_init(o_done + i, 1);
            mbar_init(o_final + i, 1);
            mbar_init(g_full + i, 1);
            mbar_init(g_empty + i, 4);
            for (int b = 0; b < 2; ++b) {
                mbar_init(s_full + 2 * i + b, 1);
                mbar_init(p_full + 2 * i + b, 128);
            }
        }
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(k_empty + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(v_empty + i, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::PRODUCER_WARP) {
        // Rows 32w+30 and 32w+31 of every Q tile are never loaded: zero them once.
        for (int x = 0; x < TILES; ++x)
            for (int c = 0; c < KCHUNKS; ++c)
                for (int i = lane; i < 4 * 2 * 8; i += 32) {
                    const int row = 32 * (i >> 4) + 30 + ((i >> 3) & 1);
                    reinterpret_cast<uint4 *>(smem + C::OFF_Q + x * Q_TILE + c * Q_CHUNK + row * 128)[i & 7] =
                        make_uint4(0, 0, 0, 0);
                }
        fence_proxy_async_smem();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::PRODUCER_WARP) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_qs);
            tma_prefetch_desc(&tm_qn);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            if constexpr (C::ASYNC_EPI) {
                tma_prefetch_desc(&tm_gate);
                tma_prefetch_desc(&tm_lam);
            }
            int kv = 0, issued_kv = 0;  // K/V tiles issued by this CTA (ring position)
            int gate_items = 0;         // items whose gate/lambda loads were issued
            int n_item = 0;
            bool ok = true;
            for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
                const Item it = item_at(w);
                for (int x = 0; x < TILES; ++x) {
                    // the previous item's last QK^T must be done before Q_x is overwritten
                    if (n_item > 0 && !mbar_wait(q_empty + x, (n_item - 1) & 1, abort_flag, ERR_SITE_PREFILL | 10)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(q_full + x, Q_TX);
                    const int row0 = it.s0 + it.t0 + x * TOK;
                    for (int c = 0; c < KCHUNKS; ++c) {
                        uint8_t *qc = smem + C::OFF_Q + x * Q_TILE + c * Q_CHUNK;
                        for (int q = 0; q < 4; ++q) {
                            tma_load_3d(qc + (32 * q) * 128, &tm_qs, q_full + x, c * 64, 4 * it.group, row0 + 6 * q);
                            tma_load_3d(qc + (32 * q + 24) * 128, &tm_qn, q_full + x, c * 64, it.group, row0 + 6 * q);
                        }
                    }
                }
                // Async epilogue: each q tile's gate logits and lambda, issued once the
                // item's first K/V tiles are on their way (the staging buffer is free
                // once the previous item's output store has read it).
                auto issue_gate = [&]() {
                    for (int x = 0; x < TILES; ++x) {
                        if (n_item > 0 && !mbar_wait(g_empty + x, (n_item - 1) & 1, abort_flag, ERR_SITE_PREFILL | 11))
                            return false;
                        mbar_arrive_expect_tx(g_full + x, C::GATE_TX);
                        const int row0 = it.s0 + it.t0 + x * TOK;
                        for (int h = 0; h < C::G_HALVES; ++h)
                            tma_load_3d(smem + C::OFF_G + (x * C::G_HALVES + h) * G_HALF, &tm_gate, g_full + x, h * 64,
                                        4 * it.group, row0);
                        tma_load_2d(smem + C::OFF_LAM + x * LAM_TILE, &tm_lam, g_full + x, 4 * it.group, row0);
                    }
                    gate_items = n_item + 1;
                    return true;
                };
                const int gate_after = min(1, it.n_tiles[TILES - 1] - 1);  // K/V tile after which to issue
                if (C::ASYNC_EPI && gate_after < 0 && !issue_gate()) {
                    ok = false;
                    break;
                }
                for (int k = 0; ok && k < it.n_tiles[TILES - 1]; ++k, ++kv) {
                    const int st = kv % STAGES;
                    const uint32_t use = static_cast<uint32_t>(kv / STAGES);
                    const int row = it.s0 + it.kv_lo + k * BN;
                    if (kv >= STAGES && !mbar_wait(k_empty + st, (use + 1) & 1, abort_flag, ERR_SITE_PREFILL | 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(k_full + st, C::K_TX);
                    for (int c = 0; c < KCHUNKS; ++c)
                        tma_load_3d(smem + C::OFF_K + st * C::K_STAGE + c * C::KV_CHUNK, &tm_k, k_full + st, c * 64,
                                    it.group, row);
                    if (kv >= STAGES && !mbar_wait(v_empty + st, (use + 1) & 1, abort_flag, ERR_SITE_PREFILL | 2)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(v_full + st, C::V_TX);
                    for (int c = 0; c < VCHUNKS; ++c)
                        tma_load_3d(smem + C::OFF_V + st * C::V_STAGE + c * C::KV_CHUNK, &tm_v, v_full + st,
                                    c * 64, it.group, row);
                    issued_kv = kv + 1;
                    if (C::ASYNC_EPI && k == gate_after && !issue_gate()) {
                        ok = false;
                        break;
                    }
                }
            }
            if (*abort_flag) {
                // Another role gave up: let this thread's copies still in flight land
                // before the CTA (and its shared memory) goes away.
                for (int k = max(0, issued_kv - STAGES); k < issued_kv; ++k) {
                    mbar_wait_cycles(k_full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
                    mbar_wait_cycles(v_full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
                }
                for (int x = 0; x < TILES; ++x) mbar_wait_cycles(q_full + x, (n_item & 1) ^ 1, 1ll << 22);
                if (C::ASYNC_EPI && gate_items > 0)
                    for (int x = 0; x < TILES; ++x) mbar_wait_cycles(g_full + x, (gate_items - 1) & 1, 1ll << 22);
            }
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------ MMA issuer --------------------------------
        // The whole warp runs this loop (converged, descriptors warp-uniform);
        // one elected lane issues the MMAs and commits. Order per key tile k:
        // S_x(k) for every q tile, then PV_x(k-1) for every q tile. S_x(k) writes
        // the S buffer that held P_x(k-2), whose PV was issued earlier (tcgen05
        // MMAs of one thread execute in issue order); across items the same
        // holds because the last PV of an item is issued before the next
        // item's first QK^T.
        const uint32_t leader = elect_one_sync();
        constexpr uint32_t idesc_s = idesc_bf16_f32(ROWS, BN, false, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(ROWS, DV, false, true);
        // Descriptors of each operand base; a byte offset `off` inside an operand
        // is added as off >> 4 to the 14-bit start-address field.
        const uint64_t q_desc0 = desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
        const uint64_t k_desc0 = desc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
        const uint64_t v_desc0 = desc_sw128(smem_u32(smem + C::OFF_V), C::KV_CHUNK, 1024);
        int kv = 0;          // K/V tiles consumed by this CTA
        int sx[TILES] = {};  // S/P steps of each q tile so far (buffer and phase)
        int n_item = 0;
        bool ok = true;
        for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
            const Item it = item_at(w);
            const int n_last = it.n_tiles[TILES - 1];
#pragma unroll
            for (int x = 0; x < TILES; ++x)
                ok = ok && mbar_wait(q_full + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 3);
            if (!__all_sync(0xffffffffu, ok)) break;
            if constexpr (C::Q_IN_TMEM) {
                // Q (staged in shared memory) -> TMEM, one 16-element K step per copy;
                // the MMAs below are issued after these copies and run after them.
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk)
                    tmem_cp_128x256b_leader(tmem + C::QT_COL0 + kk * 8,
                                            q_desc0 + (((kk >> 2) * Q_CHUNK + (kk & 3) * 32) >> 4), leader);
                umma_commit_leader(q_empty + 0, leader);  // the staging buffer may be refilled
            }
            for (int k = 0; k <= n_last; ++k) {
                if (k < n_last) {
                    const int st = (kv + k) % STAGES;
                    if (!__all_sync(0xffffffffu, mbar_wait(k_full + st, ((kv + k) / STAGES) & 1, abort_flag,
                                                           ERR_SITE_PREFILL | 4))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t k_desc = k_desc0 + static_cast<uint64_t>((st * C::K_STAGE) >> 4);
#pragma unroll
                    for (int x = 0; x < TILES; ++x) {
                        if (k >= it.n_tiles[x]) continue;
                        const int b = (sx[x] + k) & 1;
                        const uint64_t q_desc = q_desc0 + static_cast<uint64_t>((x * Q_TILE) >> 4);
                        const uint32_t d = tmem + C::S_COL0 + x * 2 * BN + b * BN;
#pragma unroll
                        for (int kk = 0; kk < DQK / 16; ++kk) {
                            const uint32_t offq = ((kk >> 2) * Q_CHUNK + (kk & 3) * 32) >> 4;
                            const uint32_t offk = ((kk >> 2) * C::KV_CHUNK + (kk & 3) * 32) >> 4;
                            if constexpr (C::Q_IN_TMEM)
                                umma_ts_leader(d, tmem + C::QT_COL0 + kk * 8, k_desc + offk, idesc_s, kk > 0, leader);
                            else
                                umma_ss_leader(d, q_desc + offq, k_desc + offk, idesc_s, kk > 0, leader);
                        }
                        umma_commit_leader(s_full + x * 2 + b, leader);
                        if (!C::Q_IN_TMEM && k == it.n_tiles[x] - 1) umma_commit_leader(q_empty + x, leader);
                    }
                    umma_commit_leader(k_empty + st, leader);
                }
                if (k >= 1) {
                    const int j = k - 1;
                    const int st = (kv + j) % STAGES;
                    if (!__all_sync(0xffffffffu, mbar_wait(v_full + st, ((kv + j) / STAGES) & 1, abort_flag,
                                                           ERR_SITE_PREFILL | 6))) {
                        ok = false;
                        break;
                    }
                    const uint64_t v_desc = v_desc0 + static_cast<uint64_t>((st * C::V_STAGE) >> 4);
#pragma unroll
                    for (int x = 0; x < TILES; ++x) {
                        if (j >= it.n_tiles[x]) continue;
                        const int step = sx[x] + j;
                        if (!__all_sync(0xffffffffu, mbar_wait(p_full + x * 2 + (step & 1), (step >> 1) & 1,
                                                               abort_flag, ERR_SITE_PREFILL | 5))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t p_tmem = tmem + C::S_COL0 + x * 2 * BN + (step & 1) * BN;
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk)
                            umma_ts_leader(tmem + C::O_COL0 + x * 128, p_tmem + kk * 8, v_desc + ((kk * 2048) >> 4),
                                           idesc_o, (j > 0 || kk > 0) ? 1u : 0u, leader);
                        umma_commit_leader(o_done + x, leader);
                        if (j == it.n_tiles[x] - 1) umma_commit_leader(o_final + x, leader);
                    }
                    if (!ok) break;
                    umma_commit_leader(v_empty + st, leader);
                }
            }
            kv += n_last;
#pragma unroll
            for (int x = 0; x < TILES; ++x) sx[x] += it.n_tiles[x];
        }
    } else {
        // --------------------------- softmax + epilogue ---------------------------
        const int x = warp >> 2;  // q tile of this warpgroup
        const int wq = warp & 3;  // TMEM lane quarter = this warp's 6 tokens
        const bool is_sig = lane < 24;
        const int tau = 6 * wq + (is_sig ? (lane >> 2) : (lane - 24));  // token in tile
        const int hsrc = 24 + (lane >> 2);  // lane holding this signal row's noise row
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t o_addr = lane_base + C::O_COL0 + x * 128;
        const float c_log2 = 0.07216878364870322f * 1.4426950408889634f;  // log2(e) / sqrt(192)
        const bool wide = ((reinterpret_cast<uintptr_t>(gate) | reinterpret_cast<uintptr_t>(out)) & 31u) == 0;
        int sxs = 0;  // S/P steps of this q tile so far
        int pv = 0;   // PV products of this q tile so far (o_done phases)
        int n_item = 0;
        bool ok = true;
        for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
            const Item it = item_at(w);
            int nt = it.n_tiles[0];
#pragma unroll
            for (int i = 1; i < TILES; ++i)
                if (x == i) nt = it.n_tiles[i];
            const int tx0 = it.t0 + x * TOK;  // first token of this tile
            const int t = tx0 + tau;
            const int lo_t = (window > 0) ? t - window + 1 : -0x40000000;
            float m_run = -INFINITY, l_run = 0.f;

            for (int k = 0; k < nt; ++k) {
                const int step = sxs + k;
                const int b = step & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(s_full + x * 2 + b, (step >> 1) & 1, abort_flag,
                                                       ERR_SITE_PREFILL | 7))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t s_addr = lane_base + C::S_COL0 + x * 2 * BN + b * BN;
                float s[BN];
#pragma unroll
                for (int h = 0; h < BN / 64; ++h) {
                    uint32_t rr[64];
                    tmem_ld64(s_addr + h * 64, rr);
#pragma unroll
                    for (int i = 0; i < 64; ++i) s[h * 64 + i] = __uint_as_float(rr[i]);
                }
                const int u0 = it.kv_lo + k * BN;
                const bool need_mask = (u0 + BN - 1 > tx0) || (window > 0 && u0 < tx0 + TOK - window);
                if (need_mask) {
                    // visible columns: keys lo_t..t of this row
                    const int c_lo = lo_t - u0, c_hi = t - u0;
#pragma unroll
                    for (int i = 0; i < BN; ++i) s[i] = (i >= c_lo && i <= c_hi) ? s[i] : -INFINITY;
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
                const uint64_t scale2 = f2_pack(c_log2, c_log2);
                const uint64_t neg_m2 = f2_pack(-mb, -mb);
                uint64_t lsum_a = f2_pack(0.f, 0.f), lsum_b = f2_pack(0.f, 0.f);
                // p = exp2(s * log2(e)/sqrt(192) - m): scaling and row sums in packed
                // fp32 pairs; one pair in kPolyEvery through the FMA-pipe polynomial,
                // the others through MUFU ex2, so both pipes share the work.
#pragma unroll
                for (int h = 0; h < BN / 64; ++h) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint64_t xx = f2_fma(f2_pack(s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]), scale2, neg_m2);
                        float p0, p1;
                        if ((i % kPolyEvery) == kPolyEvery - 1) {
                            exp2_poly_pair(xx, p0, p1);
                        } else {
                            float x0, x1;
                            f2_unpack(xx, x0, x1);
                            p0 = fast_exp2(x0);
                            p1 = fast_exp2(x1);
                        }
                        if (i & 1)
                            lsum_b = f2_add(lsum_b, f2_pack(p0, p1));
                        else
                            lsum_a = f2_add(lsum_a, f2_pack(p0, p1));
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(s_addr + h * 32, pk);
                }
                {
                    float a0, a1, b0, b1;
                    f2_unpack(lsum_a, a0, a1);
                    f2_unpack(lsum_b, b0, b1);
                    l_run += (a0 + a1) + (b0 + b1);
                }
                if (k > 0 && __any_sync(0xffffffffu, resc)) {
                    // O_x still holds PV_x(k-1)'s accumulation: wait for it, then rescale.
                    if (!__all_sync(0xffffffffu, mbar_wait(o_done + x, (pv + k - 1) & 1, abort_flag,
                                                           ERR_SITE_PREFILL | 8))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float a = resc ? alpha : 1.f;
#pragma unroll
                    for (int ch = 0; ch < DV / 32; ++ch) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + ch * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                        tmem_st32(o_addr + ch * 32, o);
                    }
                }
                tc_fence_before();
                mbar_arrive(p_full + x * 2 + b);
            }
            if (!ok) break;
            sxs += nt;
            pv += nt;

            // ----------------------------- epilogue ------------------------------
            const bool valid = is_sig && (t < it.L);
            const size_t row = static_cast<size_t>(it.s0 + t) * hs + 4 * it.group + (lane & 3);
            if constexpr (C::EPI == EPI_STAGED) {
                // Gate and lambda were staged in shared memory during the item; the
                // output replaces the gate in place and leaves by one TMA store per
                // warp and half, or (a warp with tokens past the sequence end)
                // by direct stores of its valid rows.
                const bool warp_full = (tx0 + 6 * wq + 5) < it.L;
                bool ok_w = mbar_wait(g_full + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 12);
                ok_w = ok_w && mbar_wait(o_final + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 9);
                if (!__all_sync(0xffffffffu, ok_w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
                const float lam = is_sig ? reinterpret_cast<const float *>(smem + C::OFF_LAM + x * LAM_TILE)[24 * wq + lane]
                                         : 0.f;
                const uint32_t g_base = smem_u32(smem + C::OFF_G + x * G_TILE) + (24 * wq + lane) * 128;
                // Each half (dims 0..63, 64..127) leaves by its TMA store as soon as it is
                // written, so the first half's store overlaps the second half's arithmetic.
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int ch = 2 * h + c2;
                        uint32_t o[32];
                        tmem_ld32(o_addr + ch * 32, o);
                        epi_chunk_staged(o, inv_l, lam, hsrc, is_sig, g_base + h * G_HALF, lane & 7, ch, warp_full,
                                         valid && !warp_full, out + row * DV + ch * 32);
                    }
                    if (warp_full) {
                        fence_proxy_async_smem();  // the generic writes above, before the TMA store reads them
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&tm_out, smem + C::OFF_G + x * G_TILE + h * G_HALF + wq * G_WARP_BOX, h * 64,
                                         4 * it.group, it.s0 + tx0 + 6 * wq);
                            bulk_commit_group();
                        }
                    }
                }
                if (warp_full && lane == 0) bulk_wait_group_read0();  // the staging buffer may be refilled
                __syncwarp();
                if (lane == 0) mbar_arrive(g_empty + x);
            } else if constexpr (C::EPI == EPI_HALF) {
                // Gate dims 0..63 and lambda were staged during the item; dims 64..127
                // are fetched now, while dims 0..63 are computed and stored.
                uint32_t gw[2][16];
                epi_fetch_gate(valid, row, gate, wide, 2, gw[0]);
                epi_fetch_gate(valid, row, gate, wide, 3, gw[1]);
                bool ok_w = mbar_wait(g_full + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 12);
                ok_w = ok_w && mbar_wait(o_final + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 9);
                if (!__all_sync(0xffffffffu, ok_w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
                const float lam = is_sig ? reinterpret_cast<const float *>(smem + C::OFF_LAM + x * LAM_TILE)[24 * wq + lane]
                                         : 0.f;
                const uint32_t g_base = smem_u32(smem + C::OFF_G + x * G_HALF) + (24 * wq + lane) * 128;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    uint32_t g[16];
                    epi_gate_staged(is_sig, g_base, lane & 7, ch, g);
                    uint32_t o[32];
                    tmem_ld32(o_addr + ch * 32, o);
                    epi_chunk(o, inv_l, lam, g, hsrc, valid, wide, out + row * DV + ch * 32);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(g_empty + x);  // the staged gate half has been read
#pragma unroll
                for (int ch = 2; ch < 4; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + ch * 32, o);
                    epi_chunk(o, inv_l, lam, gw[ch - 2], hsrc, valid, wide, out + row * DV + ch * 32);
                }
            } else if constexpr (C::EPI == EPI_BWD) {
                if (!__all_sync(0xffffffffu, mbar_wait(o_final + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 9))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const size_t tok = static_cast<size_t>(it.s0 + t);
                epi_backward(o_addr, l_run, m_run, is_sig, t < it.L, lane, hsrc, tok, hs, hkv, it.group, lambda, gate,
                             bwd);
            } else {
                // Signal rows fetch their gate row and lambda before waiting for the last PV.
                uint32_t gw[DV / 32][16];
#pragma unroll
                for (int ch = 0; ch < DV / 32; ++ch) epi_fetch_gate(valid, row, gate, wide, ch, gw[ch]);
                const float lam = valid ? __ldg(lambda + row) : 0.f;
                // o_final completes once per item, after this tile's last PV product.
                if (!__all_sync(0xffffffffu, mbar_wait(o_final + x, n_item & 1, abort_flag, ERR_SITE_PREFILL | 9))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll
                for (int ch = 0; ch < DV / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + ch * 32, o);
                    epi_chunk(o, inv_l, lam, gw[ch], hsrc, valid, wide, out + row * DV + ch * 32);
                }
            }
            // every lane's TMEM reads of O are complete before the next item's PV
            // products may overwrite it (they wait for this warpgroup's p_full).
            tc_fence_before();
        }
    }

    if (C::EPI == EPI_STAGED && warp < C::PRODUCER_WARP && lane == 0) bulk_wait_group0();  // output stores complete
    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------
// Full causal and windows over kPrefillSlidingMaxWindow: the one-tile configuration.
using LongCfg = pf::CausalCfg;

PrefillGeometry prefill_geometry(int window) {
    // Short windows: 48-token items over 64-key tiles; otherwise 24-token items over 128-key tiles.
    if (window > 0 && window <= kPrefillSlidingMaxWindow)
        return {pf::SlidingCfg::CTA_TOK, pf::SlidingCfg::BN, pf::SlidingCfg::V_BOX, pf::SlidingCfg::ASYNC_EPI};
    return {LongCfg::CTA_TOK, LongCfg::BN, LongCfg::V_BOX, LongCfg::ASYNC_EPI};
}

// Each kernel instantiation opts in to its shared memory once per device (a
// driver call that need not be repeated on every launch).
template <class C, class Plan>
static cudaError_t launch_cfg(const PrefillLaunch &L, const Plan &plan, int dev, int num_sms, cudaStream_t stream) {
    static PerContextFlag attr_set;  // per device, for the context it was set in
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        cudaError_t e = cudaFuncSetAttribute(gdla_prefill_kernel<C, Plan>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    const long long work = static_cast<long long>(plan.n_items) * plan.hkv;
    const unsigned grid = static_cast<unsigned>(work < num_sms ? work : num_sms);
    gdla_prefill_kernel<C, Plan><<<grid, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(
        L.tm_qs, L.tm_qn, L.tm_k, L.tm_v, L.tm_gate, L.tm_lam, L.tm_out, L.lambda, L.gate, L.out, L.bwd, plan);
    return cudaPeekAtLastError();
}

// The plan in the smallest capacity that holds it (kernel parameters are
// copied with every launch).
template <class C>
static cudaError_t launch_sized(const PrefillLaunch &L, const PrefillPlan &plan, int dev, int num_sms,
                                cudaStream_t stream) {
    auto shrink = [&](auto &small) {
        small.n_items = plan.n_items;
        small.hkv = plan.hkv;
        small.window = plan.window;
        small.n_seqs = plan.n_seqs;
        std::memcpy(small.seq_start, plan.seq_start, sizeof(int) * plan.n_seqs);
        std::memcpy(small.seq_len, plan.seq_len, sizeof(int) * plan.n_seqs);
        std::memcpy(small.items, plan.items, sizeof(uint32_t) * plan.n_items);
    };
    if (plan.n_items <= PrefillPlanSmall::kMaxItems && plan.n_seqs <= PrefillPlanSmall::kMaxSeqs) {
        PrefillPlanSmall small;
        shrink(small);
        return launch_cfg<C>(L, small, dev, num_sms, stream);
    }
    if (plan.n_items <= PrefillPlanMedium::kMaxItems && plan.n_seqs <= PrefillPlanMedium::kMaxSeqs) {
        PrefillPlanMedium medium;
        shrink(medium);
        return launch_cfg<C>(L, medium, dev, num_sms, stream);
    }
    return launch_cfg<C>(L, plan, dev, num_sms, stream);
}

cudaError_t launch_prefill_bwd_recompute(const PrefillLaunch &L, const PrefillPlan &plan, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int num_sms = device_sm_count(dev);
    if (num_sms <= 0) return cudaErrorInvalidDevice;
    if (plan.window > 0 && plan.window <= kPrefillSlidingMaxWindow)
        return launch_sized<pf::BwdRecomputeSlidingCfg>(L, plan, dev, num_sms, stream);
    return launch_sized<pf::BwdRecomputeCfg>(L, plan, dev, num_sms, stream);
}

cudaError_t launch_prefill(const PrefillLaunch &L, const PrefillPlan &plan, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int num_sms = device_sm_count(dev);
    if (num_sms <= 0) return cudaErrorInvalidDevice;
    if (plan.window > 0 && plan.window <= kPrefillSlidingMaxWindow)
        return launch_sized<pf::SlidingCfg>(L, plan, dev, num_sms, stream);
    return launch_sized<LongCfg>(L, plan, dev, num_sms, stream);
}

}  // namespace gdla
