// gdla_prefill_bwd.cu - GDLA prefill backward: the attention gradients, for sm_100a.
//
// Method (aitrends.kr/articles/94908, GDLA paragraphs: 4 signal + 1 noise
// query heads per KV group over one K_j, V_j; D = H_S - lambda H_N; sigmoid
// gate). The forward recompute (gdla_prefill.cu, backward epilogue) leaves per
// row the gradient dH of the head output H (bf16), lse2 = log2 of the softmax
// denominator in the scaled base-2 units the kernels use, and rowsum(dH * H).
// With P = exp2(S c - lse2), c = log2(e)/sqrt(192), for each head h over the
// shared K_j, V_j:
//     dP = dH V^T,   dS = P (dP - rowsum(dH H)),
//     dQ_h = dS K / sqrt(192),   dK_j = sum_h dS^T Q_h / sqrt(192),   dV_j = sum_h P^T dH_h.
// Rows keep the forward's tile layout: 24 tokens x 5 heads in the 128 lanes of
// a tile, per TMEM lane quarter w tokens 6w..6w+5 as rows 32w+4i+h (signal head
// h of token 6w+i), 32w+24+i (noise head), 32w+30..31 unused (zero).
//
// Two kernels, no atomics (deterministic):
//   dq kernel   - item (KV group, 24-token q tile), loop over its 64-key tiles:
//                 S = Q K^T and dP = dH V^T (tcgen05, M=128 rows, N=64 keys),
//                 dS by the 4 row warps into TMEM, dQ += dS K (A = dS from TMEM,
//                 B = the K tile read keys-major, N=192).
//   dkv kernel  - item (KV group, 128-key tile), loop over the 12-token halves
//                 of q tiles that see it: S^T = K Q^T and dP^T = V dH^T
//                 (M=128 keys, N=64 rows), P^T and dS^T by the 4 key warps into
//                 TMEM, dV += P^T dH and dK += dS^T Q (A from TMEM, B the row
//                 tile read rows-major).
// Each output row (dq of a token and head, dk / dv of a key) is owned by one
// CTA and written once.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "gdla_internal.h"
#include "gdla_ptx.cuh"

namespace gdla {

namespace pb {
constexpr int TOK = kPrefillTileTokens;  // 24
constexpr int DQK = 192, DV = 128;
constexpr int ROW_BOX = TOK / 4;         // 6 tokens per TMA box (one lane quarter)
constexpr uint32_t QBOX_TX = 64 * 4 * ROW_BOX * 2 + 64 * 1 * ROW_BOX * 2;  // one quarter's rows of one 64-dim chunk
constexpr float kScoreLog2 = 0.07216878364870322f * 1.4426950408889634f;  // log2(e) / sqrt(192)
constexpr float kInvRoot = 0.07216878364870322f;                         // 1 / sqrt(192)
constexpr int NUM_THREADS = 192;  // 4 row/key warps, producer warp 4, MMA warp 5
constexpr int PRODUCER_WARP = 4, MMA_WARP = 5;

// (row of a 32-row lane quarter) -> token offset in the quarter, head (0..3 signal, 4 noise), padding
__host__ __device__ constexpr int quarter_token(int within) { return within < 24 ? within >> 2 : within - 24; }
__host__ __device__ constexpr int quarter_head(int within) { return within < 24 ? (within & 3) : 4; }
}  // namespace pb

// Two 32-column TMEM loads (any two column addresses of this warp's lanes) with one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t a0, uint32_t a1, uint32_t (&r0)[32], uint32_t (&r1)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0[0]), "=r"(r0[1]), "=r"(r0[2]), "=r"(r0[3]), "=r"(r0[4]), "=r"(r0[5]), "=r"(r0[6]), "=r"(r0[7]), "=r"(r0[8]), "=r"(r0[9]), "=r"(r0[10]), "=r"(r0[11]), "=r"(r0[12]), "=r"(r0[13]), "=r"(r0[14]), "=r"(r0[15]), "=r"(r0[16]), "=r"(r0[17]), "=r"(r0[18]), "=r"(r0[19]), "=r"(r0[20]), "=r"(r0[21]), "=r"(r0[22]), "=r"(r0[23]), "=r"(r0[24]), "=r"(r0[25]), "=r"(r0[26]), "=r"(r0[27]), "=r"(r0[28]), "=r"(r0[29]), "=r"(r0[30]), "=r"(r0[31]), "=r"(r1[0]), "=r"(r1[1]), "=r"(r1[2]), "=r"(r1[3]), "=r"(r1[4]), "=r"(r1[5]), "=r"(r1[6]), "=r"(r1[7]), "=r"(r1[8]), "=r"(r1[9]), "=r"(r1[10]), "=r"(r1[11]), "=r"(r1[12]), "=r"(r1[13]), "=r"(r1[14]), "=r"(r1[15]), "=r"(r1[16]), "=r"(r1[17]), "=r"(r1[18]), "=r"(r1[19]), "=r"(r1[20]), "=r"(r1[21]), "=r"(r1[22]), "=r"(r1[23]), "=r"(r1[24]), "=r"(r1[25]), "=r"(r1[26]), "=r"(r1[27]), "=r"(r1[28]), "=r"(r1[29]), "=r"(r1[30]), "=r"(r1[31])
        : "r"(a0), "r"(a1)
        : "memory");
}
// Two 16-column TMEM stores with one wait.
__device__ __forceinline__ void tmem_st16x2(uint32_t a0, const uint32_t (&r0)[16], uint32_t a1,
                                            const uint32_t (&r1)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17};\n\t"
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%1], {%18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(a0), "r"(a1), "r"(r0[0]), "r"(r0[1]), "r"(r0[2]), "r"(r0[3]), "r"(r0[4]), "r"(r0[5]), "r"(r0[6]), "r"(r0[7]), "r"(r0[8]), "r"(r0[9]), "r"(r0[10]), "r"(r0[11]), "r"(r0[12]), "r"(r0[13]), "r"(r0[14]), "r"(r0[15]), "r"(r1[0]), "r"(r1[1]), "r"(r1[2]), "r"(r1[3]), "r"(r1[4]), "r"(r1[5]), "r"(r1[6]), "r"(r1[7]), "r"(r1[8]), "r"(r1[9]), "r"(r1[10]), "r"(r1[11]), "r"(r1[12]), "r"(r1[13]), "r"(r1[14]), "r"(r1[15])
        : "memory");
}

// ------------------------------------------------------------------------------
// dQ
// ------------------------------------------------------------------------------
namespace pbq {
using namespace pb;
constexpr int BN = 64;                     // keys per tile
constexpr int STAGES = 3;
constexpr int Q_CHUNK = 128 * 128;         // 128 rows x 64 dims
constexpr int Q_BYTES = 3 * Q_CHUNK;       // 48 KB
constexpr int DH_BYTES = 2 * Q_CHUNK;      // 32 KB
constexpr int KV_CHUNK = BN * 128;         // 64 keys x 64 dims: 8 KB
constexpr int K_STAGE = 3 * KV_CHUNK;
constexpr int V_STAGE = 2 * KV_CHUNK;
constexpr int STAGE = K_STAGE + V_STAGE;   // 40 KB
constexpr int OFF_Q = 0;
constexpr int OFF_DH = OFF_Q + Q_BYTES;
constexpr int OFF_KV = OFF_DH + DH_BYTES;
constexpr int OFF_BAR = OFF_KV + STAGES * STAGE;
constexpr int OFF_MISC = OFF_BAR + 16 * 8;
constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
constexpr uint32_t QD_TX = (3 + 2) * 4 * QBOX_TX;  // Q and dH tiles of one item
// dQ, then two buffers of (S, dP): the next key tile's products run while the
// row warps turn this tile's into dS (written over its S).
constexpr uint32_t DQ_COL = 0, S_COL0 = 192, DP_COL0 = 256, BUF_COLS = 128;
// The item's dH tile, copied from shared memory once per item: dP = dH V^T then reads
// its A operand from TMEM (only V from shared memory, full rate at N = 64).
constexpr uint32_t DH_COL = 448;
constexpr uint32_t TMEM_COLS = 512;
static_assert(DH_COL + DV / 2 <= TMEM_COLS, "TMEM budget");
// 8 row warps: two per TMEM lane quarter (warp % 4), each taking one half (warp / 4)
// of a key tile's 32 + 32 columns; producer warp 8, MMA warp 9.
constexpr int ROW_WARPS = 8;
constexpr int NUM_THREADS = 32 * ROW_WARPS + 64;
constexpr int PRODUCER_WARP = ROW_WARPS, MMA_WARP = ROW_WARPS + 1;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace pbq

template <class Plan>
__global__ void __launch_bounds__(pbq::NUM_THREADS, 1)
gdla_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_qn,
                   const __grid_constant__ CUtensorMap tm_dhs, const __grid_constant__ CUtensorMap tm_dhn,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float *__restrict__ stats, __nv_bfloat16 *__restrict__ dq_sig,
                   __nv_bfloat16 *__restrict__ dq_noise, const __grid_constant__ Plan plan) {
    using namespace pbq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *q_full = bars + 0;    // one phase per item: Q and dH tiles landed
    uint64_t *q_empty = bars + 1;   // one phase per item: its last S / dP products are done
    uint64_t *kv_full = bars + 2;   // [stage]
    uint64_t *kv_empty = bars + 5;  // [stage]
    uint64_t *s_full = bars + 8;    // [buffer]: S and dP of a key tile in TMEM
    uint64_t *ds_full = bars + 10;  // [buffer]: its dS in TMEM (one arrival per row-warp thread)
    uint64_t *dq_final = bars + 12; // one phase per item: its last dQ product is done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hkv = plan.hkv, hs = 4 * hkv, window = plan.window;
    const int n_work = plan.n_items * hkv;

    struct Item {
        int group, s0, L, t0, kv_lo, n_tiles;
    };
    auto item_at = [&](int w) {
        Item it;
        it.group = w % hkv;
        const uint32_t code = plan.items[w / hkv];
        const int seq = static_cast<int>(code >> kItemSeqShift);
        it.s0 = plan.seq_start[seq];
        it.L = plan.seq_len[seq];
        it.t0 = static_cast<int>(code & kItemTileMask) * TOK;
        it.kv_lo = (window > 0) ? max(0, it.t0 - window + 1) : 0;
        it.n_tiles = max(1, (min(it.L, it.t0 + TOK) - it.kv_lo + BN - 1) / BN);
        return it;
    };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(kv_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full + b, 1);
            mbar_init(ds_full + b, 32 * ROW_WARPS);
        }
        mbar_init(dq_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == pbq::PRODUCER_WARP) {
        // rows 32w+30, 32w+31 of the Q and dH tiles are never loaded: zero them once
        for (int c = 0; c < 5; ++c)
            for (int i = lane; i < 4 * 2 * 8; i += 32) {
                const int row = 32 * (i >> 4) + 30 + ((i >> 3) & 1);
                reinterpret_cast<uint4 *>(smem + OFF_Q + c * Q_CHUNK + row * 128)[i & 7] = make_uint4(0, 0, 0, 0);
            }
        fence_proxy_async_smem();
    }
    if (warp == pbq::MMA_WARP) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == pbq::PRODUCER_WARP) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int kv = 0, issued = 0, n_item = 0;
            bool ok = true;
            for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
                const Item it = item_at(w);
                if (n_item > 0 && !mbar_wait(q_empty, (n_item - 1) & 1, abort_flag, ERR_SITE_BWD | 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(q_full, QD_TX);
                const int row0 = it.s0 + it.t0;
                for (int q = 0; q < 4; ++q) {
                    for (int c = 0; c < 3; ++c) {
                        uint8_t *dst = smem + OFF_Q + c * Q_CHUNK + 32 * q * 128;
                        tma_load_3d(dst, &tm_qs, q_full, c * 64, 4 * it.group, row0 + 6 * q);
                        tma_load_3d(dst + 24 * 128, &tm_qn, q_full, c * 64, it.group, row0 + 6 * q);
                    }
                    for (int c = 0; c < 2; ++c) {
                        uint8_t *dst = smem + OFF_DH + c * Q_CHUNK + 32 * q * 128;
                        tma_load_3d(dst, &tm_dhs, q_full, c * 64, 4 * it.group, row0 + 6 * q);
                        tma_load_3d(dst + 24 * 128, &tm_dhn, q_full, c * 64, it.group, row0 + 6 * q);
                    }
                }
                for (int k = 0; k < it.n_tiles; ++k, ++kv) {
                    const int st = kv % STAGES;
                    if (kv >= STAGES &&
                        !mbar_wait(kv_empty + st, ((kv / STAGES) + 1) & 1, abort_flag, ERR_SITE_BWD | 2)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(kv_full + st, STAGE);
                    const int row = it.s0 + it.kv_lo + k * BN;
                    uint8_t *sb = smem + OFF_KV + st * STAGE;
                    for (int c = 0; c < 3; ++c) tma_load_3d(sb + c * KV_CHUNK, &tm_k, kv_full + st, c * 64, it.group, row);
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sb + K_STAGE + c * KV_CHUNK, &tm_v, kv_full + st, c * 64, it.group, row);
                    issued = kv + 1;
                }
            }
            if (*abort_flag) {
                for (int k = max(0, issued - STAGES); k < issued; ++k)
                    mbar_wait_cycles(kv_full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
                mbar_wait_cycles(q_full, (n_item & 1) ^ 1, 1ll << 22);
            }
        }
    } else if (warp == pbq::MMA_WARP) {
        // ------------------------------ MMA issuer --------------------------------
        // Order: S(0), dP(0); then per key tile k: S(k+1), dP(k+1) into the other
        // buffer, (dS(k) from the row warps), dQ(k). S(k+2) overwrites dS(k) only
        // after dQ(k) read it (one issuing thread, executed in order).
        const uint32_t leader = elect_one_sync();
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, BN, false, false);
        constexpr uint32_t idesc_q = idesc_bf16_f32(128, DQK, false, true);
        const uint64_t q_desc0 = desc_sw128(smem_u32(smem + OFF_Q), 16, 1024);
        const uint64_t dh_desc0 = desc_sw128(smem_u32(smem + OFF_DH), 16, 1024);
        const uint64_t kv_desc0 = desc_sw128(smem_u32(smem + OFF_KV), 16, 1024);        // K, V as B (keys x dims)
        const uint64_t kmn_desc0 = desc_sw128(smem_u32(smem + OFF_KV), KV_CHUNK, 1024);  // K as B (dims x keys)
        int kv = 0, step = 0, n_item = 0;
        bool ok = true;
        for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
            const Item it = item_at(w);
            if (!__all_sync(0xffffffffu, mbar_wait(q_full, n_item & 1, abort_flag, ERR_SITE_BWD | 3))) break;
            // dH (staged in shared memory) -> TMEM, one 16-dim K step per copy; the dP products
            // below are issued after these copies and run after them
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk)
                tmem_cp_128x256b_leader(tmem + DH_COL + kk * 8,
                                        dh_desc0 + (((kk >> 2) * Q_CHUNK + (kk & 3) * 32) >> 4), leader);
            // S and dP of key tile k (global tile index kv + k, global step step + k)
            auto issue_sdp = [&](int k) {
                const int st = (kv + k) % STAGES;
                if (!__all_sync(0xffffffffu,
                                mbar_wait(kv_full + st, ((kv + k) / STAGES) & 1, abort_flag, ERR_SITE_BWD | 4)))
                    return false;
                tc_fence_after();
                const uint32_t sbase = st * STAGE;
                const uint32_t buf = ((step + k) & 1) * BUF_COLS;
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const uint32_t offq = ((kk >> 2) * Q_CHUNK + (kk & 3) * 32) >> 4;
                    const uint32_t offk = (sbase + (kk >> 2) * KV_CHUNK + (kk & 3) * 32) >> 4;
                    umma_ss_leader(tmem + S_COL0 + buf, q_desc0 + offq, kv_desc0 + offk, idesc_s, kk > 0, leader);
                }
#pragma unroll
                for (int kk = 0; kk < DV / 16; ++kk) {
                    const uint32_t offv = (sbase + K_STAGE + (kk >> 2) * KV_CHUNK + (kk & 3) * 32) >> 4;
                    umma_ts_leader(tmem + DP_COL0 + buf, tmem + DH_COL + kk * 8, kv_desc0 + offv, idesc_s, kk > 0,
                                   leader);
                }
                umma_commit_leader(s_full + ((step + k) & 1), leader);
                if (k == it.n_tiles - 1) umma_commit_leader(q_empty, leader);
                return true;
            };
            ok = issue_sdp(0);
            for (int k = 0; ok && k < it.n_tiles; ++k) {
                if (k + 1 < it.n_tiles && !issue_sdp(k + 1)) {
                    ok = false;
                    break;
                }
                const int st = (kv + k) % STAGES;
                const int sk = step + k;
                if (!__all_sync(0xffffffffu, mbar_wait(ds_full + (sk & 1), (sk >> 1) & 1, abort_flag, ERR_SITE_BWD | 5))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sbase = st * STAGE;
                const uint32_t buf = (sk & 1) * BUF_COLS;
                // packed dS of keys 32 h .. 32 h + 31 sits in columns 32 h .. 32 h + 15 of the buffer
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_ts_leader(tmem + DQ_COL, tmem + S_COL0 + buf + (kk >> 1) * 32 + (kk & 1) * 8,
                                   kmn_desc0 + ((sbase + kk * 2048) >> 4), idesc_q, (k > 0 || kk > 0) ? 1u : 0u,
                                   leader);
                umma_commit_leader(kv_empty + st, leader);
                if (k == it.n_tiles - 1) umma_commit_leader(dq_final, leader);
            }
            kv += it.n_tiles;
            step += it.n_tiles;
        }
    } else {
        // ------------------------------ row warps ---------------------------------
        const int qw = warp & 3, half = warp >> 2;  // TMEM lane quarter, key-column half
        const bool is_sig = lane < 24;
        const int tau = 6 * qw + pb::quarter_token(lane);
        const int head = pb::quarter_head(lane);
        const bool pad_row = lane >= 30;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(qw * 32) << 16);
        int step = 0, n_item = 0;
        bool ok = true;
        for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
            const Item it = item_at(w);
            const int t = it.t0 + tau;
            const bool row_ok = !pad_row && t < it.L;
            const size_t srow = static_cast<size_t>(it.s0 + t) * hkv + it.group;  // (token, group)
            float lse2 = 0.f, drow = 0.f;
            if (row_ok) {
                lse2 = __ldg(stats + srow * kBwdStats + head);
                drow = __ldg(stats + srow * kBwdStats + 8 + head);
            }
            for (int k = 0; k < it.n_tiles; ++k, ++step) {
                const int b = step & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(s_full + b, (step >> 1) & 1, abort_flag, ERR_SITE_BWD | 6))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // this half's 32 keys: S and dP columns 32 half ..; packed dS over its first 16 S columns
                const uint32_t s_addr = lane_base + S_COL0 + b * BUF_COLS + 32 * half;
                uint32_t sr[32], dr[32];
                tmem_ld32x2(s_addr, lane_base + DP_COL0 + b * BUF_COLS + 32 * half, sr, dr);
                const int u0 = it.kv_lo + k * BN + 32 * half;
                // bit c: key u0 + c is visible to this row (c <= t - u0, and c > t - window - u0)
                const int hi = min(31, t - u0);
                const int lo = (window > 0) ? max(0, t - window - u0 + 1) : 0;
                const uint32_t vm = (!row_ok || hi < lo)
                                        ? 0u
                                        : ((hi == 31 ? 0xFFFFFFFFu : ((1u << (hi + 1)) - 1u)) & ~((1u << lo) - 1u));
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float ds2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int c = 2 * i + e;
                        const float p = fast_exp2(fmaf(__uint_as_float(sr[c]), kScoreLog2, -lse2));
                        ds2[e] = ((vm >> c) & 1u) ? p * (__uint_as_float(dr[c]) - drow) : 0.f;
                    }
                    pk[i] = pack_bf16x2(ds2[0], ds2[1]);
                }
                tmem_st16(s_addr, pk);
                tc_fence_before();
                mbar_arrive(ds_full + b);
            }
            if (!ok) break;
            if (!__all_sync(0xffffffffu, mbar_wait(dq_final, n_item & 1, abort_flag, ERR_SITE_BWD | 7))) break;
            tc_fence_after();
            __nv_bfloat16 *dst = is_sig ? dq_sig + ((static_cast<size_t>(it.s0 + t) * hs + 4 * it.group + head) * DQK)
                                        : dq_noise + srow * DQK;
#pragma unroll 1
            for (int ch = 3 * half; ch < 3 * half + 3; ++ch) {  // this half's 96 of dQ's 192 columns
                uint32_t o[32];
                tmem_ld32(lane_base + DQ_COL + ch * 32, o);
                if (row_ok) {
                    uint32_t wds[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        wds[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * kInvRoot, __uint_as_float(o[2 * i + 1]) * kInvRoot);
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + ch * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(wds[4 * i], wds[4 * i + 1], wds[4 * i + 2], wds[4 * i + 3]);
                }
            }
            // dQ is read before the next item's first dQ product overwrites it: that
            // product waits for these warps' ds_full of the next item's first tile.
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == pbq::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------
// dK, dV
// ------------------------------------------------------------------------------
namespace pbk {
using namespace pb;
constexpr int BK = 128;                    // keys per item
constexpr int HT = 12;                     // tokens per step (half a q tile: 64 rows)
constexpr int STAGES = 3;
constexpr int K_CHUNK = BK * 128;          // 128 keys x 64 dims: 16 KB
constexpr int K_BYTES = 3 * K_CHUNK;
constexpr int V_BYTES = 2 * K_CHUNK;
constexpr int H_CHUNK = 64 * 128;          // 64 rows x 64 dims: 8 KB
constexpr int QH_BYTES = 3 * H_CHUNK;
constexpr int DHH_BYTES = 2 * H_CHUNK;
constexpr int STATS_BYTES = HT * kBwdStats * 4;  // 768 B
constexpr int STAGE = QH_BYTES + DHH_BYTES + 1024;  // 41 KB (stats in the last 1 KB)
constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + K_BYTES;
constexpr int OFF_ST = OFF_V + V_BYTES;
constexpr int OFF_BAR = OFF_ST + STAGES * STAGE;
constexpr int OFF_MISC = OFF_BAR + 16 * 8;
constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
constexpr uint32_t KV_TX = K_BYTES + V_BYTES;
// A step's 64 rows: signal rows 4 j + h (token j < 12, head h < 4), noise rows 48 + j,
// padding rows 60..63; one 12-token box per 64-dim chunk and head kind.
constexpr int STEP_SIG_ROWS = 4 * HT, STEP_NOISE_ROW0 = 4 * HT, STEP_PAD_ROW0 = 5 * HT;
constexpr uint32_t STEP_TX = (3 + 2) * STEP_PAD_ROW0 * 128 + STATS_BYTES;
// dK, dV, two S^T buffers (each later holding P^T in its first 32 columns and
// dS^T in the next 32), one dP^T buffer (free again once the key warps have
// loaded it): step s+1's products run while the key warps work on step s.
constexpr uint32_t DK_COL = 0, DV_COL = 192, ST_COL0 = 320, DPT_COL = 448;
constexpr uint32_t TMEM_COLS = 512;
// 8 key warps: two per TMEM lane quarter (warp % 4), each taking one half (warp / 4)
// of a step's 64 rows; producer warp 8, MMA warp 9.
constexpr int KEY_WARPS = 8;
constexpr int NUM_THREADS = 32 * KEY_WARPS + 64;
constexpr int PRODUCER_WARP = KEY_WARPS, MMA_WARP = KEY_WARPS + 1;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace pbk

template <class Plan>
__global__ void __launch_bounds__(pbk::NUM_THREADS, 1)
gdla_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_qn,
                    const __grid_constant__ CUtensorMap tm_dhs, const __grid_constant__ CUtensorMap tm_dhn,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_stats, __nv_bfloat16 *__restrict__ dk,
                    __nv_bfloat16 *__restrict__ dv, const __grid_constant__ Plan plan) {
    using namespace pbk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *kv_full = bars + 0;    // one phase per item: the K and V tiles landed
    uint64_t *kv_empty = bars + 1;   // one phase per item: its last products are done
    uint64_t *st_full = bars + 2;    // [stage]: Q, dH halves and row statistics of a step
    uint64_t *st_empty = bars + 5;   // [stage]
    uint64_t *s_full = bars + 8;     // [buffer]: S^T and dP^T of a step in TMEM
    uint64_t *dpt_free = bars + 10;  // one phase per step: its dP^T has been loaded (every key-warp thread)
    uint64_t *pds_full = bars + 11;  // [buffer]: P^T and dS^T in TMEM (every key-warp thread)
    uint64_t *dkv_final = bars + 13; // one phase per item
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hkv = plan.hkv, window = plan.window;
    const int n_work = plan.n_items * hkv;

    // Item: keys u0..u0+127 of one sequence; steps: 12-token halves from u0 to the
    // last token that sees one of the keys.
    struct Item {
        int group, s0, L, u0, n_steps;
    };
    auto item_at = [&](int w) {
        Item it;
        it.group = w % hkv;
        const uint32_t code = plan.items[w / hkv];
        const int seq = static_cast<int>(code >> kItemSeqShift);
        it.s0 = plan.seq_start[seq];
        it.L = plan.seq_len[seq];
        it.u0 = static_cast<int>(code & kItemTileMask) * BK;
        const int t_end = (window > 0) ? min(it.L, it.u0 + BK - 1 + window) : it.L;
        it.n_steps = max(1, (t_end - it.u0 + HT - 1) / HT);
        return it;
    };

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_empty, 1);
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(st_full + i, 1);
            mbar_init(st_empty + i, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full + b, 1);
            mbar_init(pds_full + b, 32 * KEY_WARPS);
        }
        mbar_init(dpt_free, 32 * KEY_WARPS);
        mbar_init(dkv_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == pbk::PRODUCER_WARP) {
        // rows 60..63 of every stage's Q and dH chunks are never loaded: zero them once
        for (int st = 0; st < STAGES; ++st)
            for (int c = 0; c < 5; ++c)
                for (int i = lane; i < (64 - STEP_PAD_ROW0) * 8; i += 32)
                    reinterpret_cast<uint4 *>(smem + OFF_ST + st * STAGE + c * H_CHUNK +
                                              (STEP_PAD_ROW0 + (i >> 3)) * 128)[i & 7] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == pbk::MMA_WARP) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == pbk::PRODUCER_WARP) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int g = 0, issued = 0, n_item = 0;
            bool ok = true;
            for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
                const Item it = item_at(w);
                if (n_item > 0 && !mbar_wait(kv_empty, (n_item - 1) & 1, abort_flag, ERR_SITE_BWD | 11)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(kv_full, KV_TX);
                for (int c = 0; c < 3; ++c)
                    tma_load_3d(smem + OFF_K + c * K_CHUNK, &tm_k, kv_full, c * 64, it.group, it.s0 + it.u0);
                for (int c = 0; c < 2; ++c)
                    tma_load_3d(smem + OFF_V + c * K_CHUNK, &tm_v, kv_full, c * 64, it.group, it.s0 + it.u0);
                for (int s = 0; s < it.n_steps; ++s, ++g) {
                    const int st = g % STAGES;
                    if (g >= STAGES && !mbar_wait(st_empty + st, ((g / STAGES) + 1) & 1, abort_flag, ERR_SITE_BWD | 12)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(st_full + st, STEP_TX);
                    uint8_t *sb = smem + OFF_ST + st * STAGE;
                    const int th = it.s0 + it.u0 + s * HT;
                    for (int c = 0; c < 3; ++c) {
                        uint8_t *dst = sb + c * H_CHUNK;
                        tma_load_3d(dst, &tm_qs, st_full + st, c * 64, 4 * it.group, th);
                        tma_load_3d(dst + STEP_NOISE_ROW0 * 128, &tm_qn, st_full + st, c * 64, it.group, th);
                    }
                    for (int c = 0; c < 2; ++c) {
                        uint8_t *dst = sb + QH_BYTES + c * H_CHUNK;
                        tma_load_3d(dst, &tm_dhs, st_full + st, c * 64, 4 * it.group, th);
                        tma_load_3d(dst + STEP_NOISE_ROW0 * 128, &tm_dhn, st_full + st, c * 64, it.group, th);
                    }
                    tma_load_3d(sb + QH_BYTES + DHH_BYTES, &tm_stats, st_full + st, 0, it.group, th);
                    issued = g + 1;
                }
            }
            if (*abort_flag) {
                for (int k = max(0, issued - STAGES); k < issued; ++k)
                    mbar_wait_cycles(st_full + k % STAGES, (k / STAGES) & 1, 1ll << 22);
                mbar_wait_cycles(kv_full, (n_item & 1) ^ 1, 1ll << 22);
            }
        }
    } else if (warp == pbk::MMA_WARP) {
        // ------------------------------ MMA issuer --------------------------------
        const uint32_t leader = elect_one_sync();
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
        constexpr uint32_t idesc_v = idesc_bf16_f32(128, DV, false, true);
        constexpr uint32_t idesc_k = idesc_bf16_f32(128, DQK, false, true);
        const uint64_t k_desc0 = desc_sw128(smem_u32(smem + OFF_K), 16, 1024);
        const uint64_t v_desc0 = desc_sw128(smem_u32(smem + OFF_V), 16, 1024);
        const uint64_t st_desc0 = desc_sw128(smem_u32(smem + OFF_ST), 16, 1024);        // Q, dH halves as B (rows x dims)
        const uint64_t stmn_desc0 = desc_sw128(smem_u32(smem + OFF_ST), H_CHUNK, 1024);  // as B (dims x rows)
        // Order: S^T(0), dP^T(0); then per step s: S^T(s+1) into the other buffer,
        // (dP^T(s) loaded by the key warps) dP^T(s+1), (P^T(s), dS^T(s) written)
        // dV(s), dK(s). S^T(s+2) overwrites step s's P^T / dS^T only after dV(s) and
        // dK(s) read them (one issuing thread, executed in order).
        int g = 0, n_item = 0;
        bool ok = true;
        for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
            const Item it = item_at(w);
            if (!__all_sync(0xffffffffu, mbar_wait(kv_full, n_item & 1, abort_flag, ERR_SITE_BWD | 13))) break;
            auto issue_st = [&](int s) {  // S^T of step s (global step g + s), after its stage landed
                const int gs = g + s, st = gs % STAGES;
                if (!__all_sync(0xffffffffu, mbar_wait(st_full + st, (gs / STAGES) & 1, abort_flag, ERR_SITE_BWD | 14)))
                    return false;
                tc_fence_after();
                const uint32_t sbase = st * STAGE;
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const uint32_t offk = ((kk >> 2) * K_CHUNK + (kk & 3) * 32) >> 4;
                    const uint32_t offq = (sbase + (kk >> 2) * H_CHUNK + (kk & 3) * 32) >> 4;
                    umma_ss_leader(tmem + ST_COL0 + (gs & 1) * 64, k_desc0 + offk, st_desc0 + offq, idesc_s, kk > 0,
                                   leader);
                }
                return true;
            };
            auto issue_dpt = [&](int s) {  // dP^T of step s, then signal both products
                const int gs = g + s, st = gs % STAGES;
                const uint32_t sbase = st * STAGE;
#pragma unroll
                for (int kk = 0; kk < DV / 16; ++kk) {
                    const uint32_t offv = ((kk >> 2) * K_CHUNK + (kk & 3) * 32) >> 4;
                    const uint32_t offd = (sbase + QH_BYTES + (kk >> 2) * H_CHUNK + (kk & 3) * 32) >> 4;
                    umma_ss_leader(tmem + DPT_COL, v_desc0 + offv, st_desc0 + offd, idesc_s, kk > 0, leader);
                }
                umma_commit_leader(s_full + (gs & 1), leader);
            };
            ok = issue_st(0);
            if (ok) issue_dpt(0);
            for (int s = 0; ok && s < it.n_steps; ++s) {
                const int gs = g + s, st = gs % STAGES;
                if (s + 1 < it.n_steps) {
                    if (!issue_st(s + 1) ||
                        !__all_sync(0xffffffffu, mbar_wait(dpt_free, gs & 1, abort_flag, ERR_SITE_BWD | 18))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_dpt(s + 1);
                }
                if (!__all_sync(0xffffffffu,
                                mbar_wait(pds_full + (gs & 1), (gs >> 1) & 1, abort_flag, ERR_SITE_BWD | 15))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sbase = st * STAGE;
                const uint32_t pcol = ST_COL0 + (gs & 1) * 64;
                // rows 32 h .. 32 h + 31 of the step: packed P^T in columns 32 h .. 32 h + 15,
                // packed dS^T in 32 h + 16 .. 32 h + 31
#pragma unroll
                for (int kk = 0; kk < 64 / 16; ++kk) {
                    const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                    const uint32_t pc = pcol + (kk >> 1) * 32 + (kk & 1) * 8;
                    umma_ts_leader(tmem + DV_COL, tmem + pc, stmn_desc0 + ((sbase + QH_BYTES + kk * 2048) >> 4),
                                   idesc_v, acc, leader);
                    umma_ts_leader(tmem + DK_COL, tmem + pc + 16, stmn_desc0 + ((sbase + kk * 2048) >> 4), idesc_k,
                                   acc, leader);
                }
                umma_commit_leader(st_empty + st, leader);
            }
            if (!ok) break;
            g += it.n_steps;
            umma_commit_leader(kv_empty, leader);
            umma_commit_leader(dkv_final, leader);
        }
    } else {
        // ------------------------------ key warps ---------------------------------
        const int qw = warp & 3, half = warp >> 2;  // TMEM lane quarter, half of the step's rows
        const int kl = qw * 32 + lane;              // key of the tile = TMEM lane
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(qw * 32) << 16);
        int g = 0, n_item = 0;
        bool ok = true;
        for (int w = snake_item(0); ok && w < n_work; w = snake_item(n_item + 1), ++n_item) {
            const Item it = item_at(w);
            const int u = it.u0 + kl;
            const bool key_ok = u < it.L;
            for (int s = 0; s < it.n_steps; ++s, ++g) {
                const int st = g % STAGES, b = g & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(s_full + b, (g >> 1) & 1, abort_flag, ERR_SITE_BWD | 16))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // this half's 32 rows: S^T and dP^T columns 32 half ..; packed P^T and dS^T over them
                const uint32_t s_addr = lane_base + ST_COL0 + b * 64 + 32 * half;
                uint32_t sr[32], dr[32];
                tmem_ld32x2(s_addr, lane_base + DPT_COL + 32 * half, sr, dr);
                tc_fence_before();
                mbar_arrive(dpt_free);  // dP^T is in registers: the next step's may overwrite it
                // the step's 12 tokens: which of them see this key, and their row statistics
                const float *stat = reinterpret_cast<const float *>(smem + OFF_ST + st * STAGE + QH_BYTES + DHH_BYTES);
                const int th = it.u0 + s * HT;  // first token of the step
                uint32_t tm = 0;                // bit j: token th + j sees key u
#pragma unroll
                for (int j = 0; j < HT; ++j) {
                    const int t = th + j;
                    tm |= (key_ok && u <= t && t < it.L && (window <= 0 || t < u + window)) ? (1u << j) : 0u;
                }
                // signal rows 4j + h of the tokens j0 .. j0 + nj - 1 (h < 4), packed into pk/dk2 from 2 p0
                auto signal_rows = [&](int j0, int nj, int r0, int p0, uint32_t (&pk)[16], uint32_t (&dk2)[16]) {
#pragma unroll
                    for (int jj = 0; jj < nj; ++jj) {
                        const int j = j0 + jj;
                        const float4 L = *reinterpret_cast<const float4 *>(stat + j * kBwdStats);
                        const float4 D = *reinterpret_cast<const float4 *>(stat + j * kBwdStats + 8);
                        const bool vj = (tm >> j) & 1u;
                        const float lv[4] = {L.x, L.y, L.z, L.w}, dv[4] = {D.x, D.y, D.z, D.w};
                        float pv[4], ds[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const int r = r0 + 4 * jj + h;
                            const float p = fast_exp2(fmaf(__uint_as_float(sr[r]), kScoreLog2, -lv[h]));
                            pv[h] = vj ? p : 0.f;
                            ds[h] = vj ? p * (__uint_as_float(dr[r]) - dv[h]) : 0.f;
                        }
                        pk[p0 + 2 * jj] = pack_bf16x2(pv[0], pv[1]);
                        pk[p0 + 2 * jj + 1] = pack_bf16x2(pv[2], pv[3]);
                        dk2[p0 + 2 * jj] = pack_bf16x2(ds[0], ds[1]);
                        dk2[p0 + 2 * jj + 1] = pack_bf16x2(ds[2], ds[3]);
                    }
                };
                uint32_t pk[16], dk2[16];
                if (half == 0) {
                    signal_rows(0, 8, 0, 0, pk, dk2);  // rows 0..31: tokens 0..7
                } else {
                    signal_rows(8, 4, 0, 0, pk, dk2);  // rows 32..47: tokens 8..11
                    // rows 48..59: the noise head of tokens 0..11; rows 60..63 are padding
#pragma unroll
                    for (int m = 0; m < 6; ++m) {
                        float pv[2], ds[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = 2 * m + e;
                            const bool vj = (tm >> j) & 1u;
                            const float p = fast_exp2(fmaf(__uint_as_float(sr[16 + j]), kScoreLog2,
                                                           -stat[j * kBwdStats + 4]));
                            pv[e] = vj ? p : 0.f;
                            ds[e] = vj ? p * (__uint_as_float(dr[16 + j]) - stat[j * kBwdStats + 12]) : 0.f;
                        }
                        pk[8 + m] = pack_bf16x2(pv[0], pv[1]);
                        dk2[8 + m] = pack_bf16x2(ds[0], ds[1]);
                    }
                    pk[14] = pk[15] = 0u;
                    dk2[14] = dk2[15] = 0u;
                }
                tmem_st16x2(s_addr, pk, s_addr + 16, dk2);
                tc_fence_before();
                mbar_arrive(pds_full + b);
            }
            if (!ok) break;
            if (!__all_sync(0xffffffffu, mbar_wait(dkv_final, n_item & 1, abort_flag, ERR_SITE_BWD | 17))) break;
            tc_fence_after();
            const size_t krow = static_cast<size_t>(it.s0 + u) * hkv + it.group;
            // dK's 6 and dV's 4 32-column chunks: half 0 takes dK 0..4, half 1 dK 5 and dV 0..3
#pragma unroll 1
            for (int ch = 5 * half; ch < (half ? DQK / 32 : 5); ++ch) {
                uint32_t o[32];
                tmem_ld32(lane_base + DK_COL + ch * 32, o);
                if (key_ok) {
                    uint32_t wd[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        wd[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * kInvRoot, __uint_as_float(o[2 * i + 1]) * kInvRoot);
                    uint4 *d4 = reinterpret_cast<uint4 *>(dk + krow * DQK + ch * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(wd[4 * i], wd[4 * i + 1], wd[4 * i + 2], wd[4 * i + 3]);
                }
            }
#pragma unroll 1
            for (int ch = 0; ch < (half ? DV / 32 : 0); ++ch) {
                uint32_t o[32];
                tmem_ld32(lane_base + DV_COL + ch * 32, o);
                if (key_ok) {
                    uint32_t wd[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        wd[i] = pack_bf16x2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
                    uint4 *d4 = reinterpret_cast<uint4 *>(dv + krow * DV + ch * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(wd[4 * i], wd[4 * i + 1], wd[4 * i + 2], wd[4 * i + 3]);
                }
            }
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == pbk::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------
template <class Plan>
static cudaError_t launch_dq_sized(const BwdLaunch &L, const Plan &plan, cudaStream_t stream) {
    static PerContextFlag attr_set;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int num_sms = device_sm_count(dev);
    if (num_sms <= 0) return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        e = cudaFuncSetAttribute(gdla_bwd_dq_kernel<Plan>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 pbq::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    const long long work = static_cast<long long>(plan.n_items) * plan.hkv;
    const unsigned grid = static_cast<unsigned>(work < num_sms ? work : num_sms);
    gdla_bwd_dq_kernel<Plan><<<grid, pbq::NUM_THREADS, pbq::SMEM_BYTES, stream>>>(
        L.tm_qs, L.tm_qn, L.tm_dhs, L.tm_dhn, L.tm_k64, L.tm_v64, L.stats, L.dq_sig, L.dq_noise, plan);
    return cudaPeekAtLastError();
}

template <class Plan>
static cudaError_t launch_dkv_sized(const BwdLaunch &L, const Plan &plan, cudaStream_t stream) {
    static PerContextFlag attr_set;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int num_sms = device_sm_count(dev);
    if (num_sms <= 0) return cudaErrorInvalidDevice;
    const unsigned long long ctx = current_context_id();
    if (!attr_set.is_set(dev, ctx)) {
        e = cudaFuncSetAttribute(gdla_bwd_dkv_kernel<Plan>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 pbk::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.set(dev, current_context_id());
    }
    const long long work = static_cast<long long>(plan.n_items) * plan.hkv;
    const unsigned grid = static_cast<unsigned>(work < num_sms ? work : num_sms);
    gdla_bwd_dkv_kernel<Plan><<<grid, pbk::NUM_THREADS, pbk::SMEM_BYTES, stream>>>(
        L.tm_qs12, L.tm_qn12, L.tm_dhs12, L.tm_dhn12, L.tm_k128, L.tm_v128, L.tm_stats, L.dk, L.dv, plan);
    return cudaPeekAtLastError();
}

// The plan in the smallest capacity that holds it (kernel parameters are copied
// with every launch).
template <class F>
static cudaError_t with_sized_plan(const PrefillPlan &plan, F &&launch) {
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
        return launch(small);
    }
    if (plan.n_items <= PrefillPlanMedium::kMaxItems && plan.n_seqs <= PrefillPlanMedium::kMaxSeqs) {
        PrefillPlanMedium medium;
        shrink(medium);
        return launch(medium);
    }
    return launch(plan);
}

cudaError_t launch_bwd_dq(const BwdLaunch &L, const PrefillPlan &plan, cudaStream_t stream) {
    return with_sized_plan(plan, [&](const auto &p) { return launch_dq_sized(L, p, stream); });
}

cudaError_t launch_bwd_dkv(const BwdLaunch &L, const PrefillPlan &plan, cudaStream_t stream) {
    return with_sized_plan(plan, [&](const auto &p) { return launch_dkv_sized(L, p, stream); });
}

}  // namespace gdla
