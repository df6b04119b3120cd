// gdla_api.cu - the C ABI declared in include/gdla.h: argument checks, the
// prefill tile plan, the decode split plan, TMA tensor maps and the launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <memory>
#include <mutex>
#include <vector>

#include "gdla.h"
#include "gdla_internal.h"
#include "gdla_prologue.h"
#include "gdla_ptx.cuh"

namespace gdla {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 contiguous), 128-byte swizzled boxes.
bool make_map(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1,
              uint32_t b2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor [d1][d0] (d0 contiguous), unswizzled boxes.
bool make_map_f32_2d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint32_t b0, uint32_t b1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {d0 * 4};
    cuuint32_t box[2] = {b0, b1};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 tensor [d2][d1][d0] (d0 contiguous), unswizzled boxes.
bool make_map_f32_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                     uint32_t b1, uint32_t b2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 4, d0 * d1 * 4};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

unsigned long long current_context_id() {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    if (get_current == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    unsigned long long id = 0;
    return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

int device_sm_count(int dev) {
    static std::atomic<int> sms[kMaxCachedDevices];
    int n = 0;
    if (dev < 0 || dev >= kMaxCachedDevices)
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : 0;
    n = sms[dev].load(std::memory_order_relaxed);
    if (n == 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        sms[dev].store(n, std::memory_order_relaxed);
    return n;
}

namespace {

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct TileItem {
    int cost;  // key tiles the q-tile visits
    int seq;
    int qt;
};

// Every (sequence, unit) of `unit_tokens` tokens with its cost (cost(L, unit)),
// heaviest first, in plans of at most kPlanMaxItems units and kPlanMaxSeqs
// sequences; launch(plan) for each. Returns false on the first failed launch.
template <class Cost, class Launch>
bool run_plans(int batch, const int32_t *seqlens, int hkv, int window, int unit_tokens, Cost cost, Launch launch) {
    std::vector<TileItem> items;
    std::vector<int> seq_start(batch);
    long long s0 = 0;
    for (int b = 0; b < batch; ++b) {
        seq_start[b] = static_cast<int>(s0);
        const int L = seqlens[b];
        s0 += L;
        const int nu = (L + unit_tokens - 1) / unit_tokens;
        for (int u = 0; u < nu; ++u) items.push_back({cost(L, u), b, u});
    }
    std::stable_sort(items.begin(), items.end(), [](const TileItem &a, const TileItem &b) {
        if (a.cost != b.cost) return a.cost > b.cost;
        if (a.seq != b.seq) return a.seq < b.seq;
        return a.qt > b.qt;
    });
    std::unique_ptr<PrefillPlan> plan(new PrefillPlan);  // filled up to n_items / n_seqs, the rest unread
    std::vector<int> local(batch, -1);
    size_t pos = 0;
    while (pos < items.size()) {
        PrefillPlan &P = *plan;
        P.n_items = 0;
        P.hkv = hkv;
        P.window = window;
        int n_seq = 0;
        std::vector<int> used;
        while (pos < items.size() && P.n_items < kPlanMaxItems) {
            const TileItem &it = items[pos];
            if (local[it.seq] < 0) {
                if (n_seq == kPlanMaxSeqs) break;
                local[it.seq] = n_seq;
                P.seq_start[n_seq] = seq_start[it.seq];
                P.seq_len[n_seq] = seqlens[it.seq];
                used.push_back(it.seq);
                ++n_seq;
            }
            P.items[P.n_items++] = (static_cast<uint32_t>(local[it.seq]) << kItemSeqShift) |
                                   static_cast<uint32_t>(it.qt);
            ++pos;
        }
        for (int s : used) local[s] = -1;
        P.n_seqs = n_seq;
        if (!launch(P)) return false;
    }
    return true;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of the backward: dH of the signal and noise heads (bf16) and the row statistics.
struct BwdWorkspace {
    size_t dh_sig, dh_noise, stats, total;
};
BwdWorkspace bwd_workspace(long long n, int hkv) {
    BwdWorkspace w;
    w.dh_sig = 0;
    w.dh_noise = align256(static_cast<size_t>(n) * 4 * hkv * 128 * 2);
    w.stats = w.dh_noise + align256(static_cast<size_t>(n) * hkv * 128 * 2);
    w.total = w.stats + align256(static_cast<size_t>(n) * hkv * kBwdStats * 4);
    return w;
}

}  // namespace

DecodePlan make_decode_plan(int batch, int hkv, int max_seqlen_k, int window, int num_cache_rows) {
    DecodePlan p{};
    p.batch = batch;
    p.hkv = hkv;
    p.window = window;
    p.max_seqlen_k = max_seqlen_k;
    p.num_cache_rows = num_cache_rows;
    const int eff = (window > 0) ? std::min(window, max_seqlen_k) : max_seqlen_k;
    int ns = std::max(1, (eff + kDecodeMinSplitKeys - 1) / kDecodeMinSplitKeys);
    ns = std::min(ns, kDecodeMaxSplits);
    int keys = (eff + ns - 1) / ns;
    keys = (keys + 63) / 64 * 64;
    p.split_keys = keys;
    p.num_splits = (eff + keys - 1) / keys;
    p.ml_offset_floats = static_cast<long long>(batch) * hkv * p.num_splits * 5 * 128;
    return p;
}

// Keys per K/V TMA box of the decode kernel that runs this plan (gdla_decode.cu).
int decode_key_tile(const DecodePlan &plan);

size_t decode_workspace_bytes(const DecodePlan &p) {
    if (p.num_splits <= 1) return 0;
    return static_cast<size_t>(p.batch) * p.hkv * p.num_splits * 5 * (128 + 2) * sizeof(float);
}

}  // namespace gdla

using namespace gdla;

extern "C" {

gdla_status_t gdla_attn_fwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
                            const float *lambda, const void *gate_logits, void *out, int batch,
                            const int32_t *seqlens, int num_kv_heads, int window, void *stream) {
    if (batch < 1 || seqlens == nullptr) return GDLA_ERR_INVALID_ARG;
    if (num_kv_heads < 1 || num_kv_heads > GDLA_MAX_KV_HEADS) return GDLA_ERR_UNSUPPORTED;
    long long n_total = 0;
    for (int b = 0; b < batch; ++b) {
        if (seqlens[b] < 0) return GDLA_ERR_INVALID_ARG;
        n_total += seqlens[b];
    }
    if (n_total >= (1ll << 31)) return GDLA_ERR_INVALID_ARG;
    if (n_total == 0) return GDLA_OK;
    if (!aligned16(q_sig) || !aligned16(q_noise) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) ||
        !aligned16(gate_logits) || !aligned16(out))
        return GDLA_ERR_INVALID_ARG;

    const int hkv = num_kv_heads;
    const PrefillGeometry geo = prefill_geometry(window);
    const int T = geo.cta_tokens;
    // ---- tile plan: every (sequence, q-tile), heaviest first ----
    std::vector<TileItem> items;
    std::vector<int> seq_start(batch);
    {
        long long s0 = 0;
        for (int b = 0; b < batch; ++b) {
            seq_start[b] = static_cast<int>(s0);
            const int L = seqlens[b];
            s0 += L;
            const int nqt = (L + T - 1) / T;
            for (int qt = 0; qt < nqt; ++qt) {
                const int t0 = qt * T;
                const int lo = (window > 0) ? std::max(0, t0 - window + 1) : 0;
                const int hi = std::min(L, t0 + T);
                items.push_back({(hi - lo + geo.key_tile - 1) / geo.key_tile, b, qt});
            }
        }
    }
    std::stable_sort(items.begin(), items.end(), [](const TileItem &a, const TileItem &b) {
        if (a.cost != b.cost) return a.cost > b.cost;
        if (a.seq != b.seq) return a.seq < b.seq;
        return a.qt > b.qt;
    });

    PrefillLaunch L{};
    const uint64_t N = static_cast<uint64_t>(n_total);
    // Q boxes: the 6 tokens one warp (TMEM lane quarter) owns in an MMA tile.
    const int TQ = kPrefillTileTokens / 4;
    if (!make_map(&L.tm_qs, q_sig, 192, 4 * hkv, N, 64, 4, TQ) ||
        !make_map(&L.tm_qn, q_noise, 192, hkv, N, 64, 1, TQ) ||
        !make_map(&L.tm_k, k, 192, hkv, N, 64, 1, geo.key_tile) ||
        !make_map(&L.tm_v, v, 128, hkv, N, 64, 1, geo.v_box))
        return GDLA_ERR_CUDA;
    // The asynchronous epilogue (short windows) moves the gate logits and lambda
    // of a 24-token tile's 4 signal heads in, and each warp's 6 output tokens out.
    if (geo.async_epilogue &&
        (!make_map(&L.tm_gate, gate_logits, 128, 4 * hkv, N, 64, 4, kPrefillTileTokens) ||
         !make_map_f32_2d(&L.tm_lam, lambda, 4 * hkv, N, 4, kPrefillTileTokens) ||
         !make_map(&L.tm_out, out, 128, 4 * hkv, N, 64, 4, TQ)))
        return GDLA_ERR_CUDA;
    L.lambda = lambda;
    L.gate = static_cast<const __nv_bfloat16 *>(gate_logits);
    L.out = static_cast<__nv_bfloat16 *>(out);

    std::unique_ptr<PrefillPlan> plan(new PrefillPlan);  // filled up to n_items / n_seqs, the rest unread
    std::vector<int> local(batch, -1);
    size_t pos = 0;
    while (pos < items.size()) {
        PrefillPlan &P = *plan;
        P.n_items = 0;
        P.hkv = hkv;
        P.window = window;
        int n_seq = 0;
        std::vector<int> used;
        while (pos < items.size() && P.n_items < kPlanMaxItems) {
            const TileItem &it = items[pos];
            if (local[it.seq] < 0) {
                if (n_seq == kPlanMaxSeqs) break;
                local[it.seq] = n_seq;
                P.seq_start[n_seq] = seq_start[it.seq];
                P.seq_len[n_seq] = seqlens[it.seq];
                used.push_back(it.seq);
                ++n_seq;
            }
            P.items[P.n_items++] = (static_cast<uint32_t>(local[it.seq]) << kItemSeqShift) |
                                   static_cast<uint32_t>(it.qt);
            ++pos;
        }
        for (int s : used) local[s] = -1;
        P.n_seqs = n_seq;
        if (launch_prefill(L, P, static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDLA_ERR_CUDA;
    }
    return GDLA_OK;
}

size_t gdla_attn_bwd_workspace_bytes(long long total_tokens, int num_kv_heads) {
    if (total_tokens < 0 || total_tokens >= (1ll << 31) || num_kv_heads < 1 || num_kv_heads > GDLA_MAX_KV_HEADS)
        return 0;
    return bwd_workspace(total_tokens, num_kv_heads).total;
}

gdla_status_t gdla_attn_bwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
                            const float *lambda, const void *gate_logits, const void *dout, void *dq_sig,
                            void *dq_noise, void *dk, void *dv, float *dlambda, void *dgate, int batch,
                            const int32_t *seqlens, int num_kv_heads, int window, void *workspace,
                            size_t workspace_bytes, void *stream) {
    if (batch < 1 || seqlens == nullptr) return GDLA_ERR_INVALID_ARG;
    if (num_kv_heads < 1 || num_kv_heads > GDLA_MAX_KV_HEADS) return GDLA_ERR_UNSUPPORTED;
    long long n_total = 0;
    for (int b = 0; b < batch; ++b) {
        if (seqlens[b] < 0) return GDLA_ERR_INVALID_ARG;
        n_total += seqlens[b];
    }
    if (n_total >= (1ll << 31)) return GDLA_ERR_INVALID_ARG;
    if (n_total == 0) return GDLA_OK;
    if (!aligned16(q_sig) || !aligned16(q_noise) || !aligned16(k) || !aligned16(v) || !aligned16(lambda) ||
        !aligned16(gate_logits) || !aligned16(dout) || !aligned16(dq_sig) || !aligned16(dq_noise) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(dlambda) || !aligned16(dgate))
        return GDLA_ERR_INVALID_ARG;
    const int hkv = num_kv_heads;
    const BwdWorkspace ws = bwd_workspace(n_total, hkv);
    if (workspace == nullptr || workspace_bytes < ws.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return GDLA_ERR_WORKSPACE;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    __nv_bfloat16 *dh_sig = reinterpret_cast<__nv_bfloat16 *>(wsb + ws.dh_sig);
    __nv_bfloat16 *dh_noise = reinterpret_cast<__nv_bfloat16 *>(wsb + ws.dh_noise);
    float *stats = reinterpret_cast<float *>(wsb + ws.stats);
    const uint64_t N = static_cast<uint64_t>(n_total);
    const int TQ = kPrefillTileTokens / 4;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // 1. forward recompute: dgate, dlambda, dH, row statistics, with the forward's tiling
    //    (24-token items over 128-key tiles; short windows 48-token items over 64-key tiles)
    const PrefillGeometry geo = prefill_geometry(window);
    PrefillLaunch F{};
    if (!make_map(&F.tm_qs, q_sig, 192, 4 * hkv, N, 64, 4, TQ) || !make_map(&F.tm_qn, q_noise, 192, hkv, N, 64, 1, TQ) ||
        !make_map(&F.tm_k, k, 192, hkv, N, 64, 1, geo.key_tile) ||
        !make_map(&F.tm_v, v, 128, hkv, N, 64, 1, geo.v_box))
        return GDLA_ERR_CUDA;
    F.lambda = lambda;
    F.gate = static_cast<const __nv_bfloat16 *>(gate_logits);
    F.bwd = {static_cast<const __nv_bfloat16 *>(dout), static_cast<__nv_bfloat16 *>(dgate), dlambda, dh_sig, dh_noise,
             stats};
    auto q_cost = [&](int T, int key_tile) {
        return [=](int L, int qt) {
            const int t0 = qt * T;
            const int lo = (window > 0) ? std::max(0, t0 - window + 1) : 0;
            return (std::min(L, t0 + T) - lo + key_tile - 1) / key_tile;
        };
    };
    if (!run_plans(batch, seqlens, hkv, window, geo.cta_tokens, q_cost(geo.cta_tokens, geo.key_tile),
                   [&](const PrefillPlan &P) { return launch_prefill_bwd_recompute(F, P, st) == cudaSuccess; }))
        return GDLA_ERR_CUDA;
    const int T = kPrefillTileTokens;

    // 2. dQ (24-token items over 64-key tiles) and 3. dK, dV (128-key items over 12-token steps)
    BwdLaunch B{};
    if (!make_map(&B.tm_qs, q_sig, 192, 4 * hkv, N, 64, 4, TQ) || !make_map(&B.tm_qn, q_noise, 192, hkv, N, 64, 1, TQ) ||
        !make_map(&B.tm_dhs, dh_sig, 128, 4 * hkv, N, 64, 4, TQ) ||
        !make_map(&B.tm_dhn, dh_noise, 128, hkv, N, 64, 1, TQ) ||
        !make_map(&B.tm_qs12, q_sig, 192, 4 * hkv, N, 64, 4, kBwdStepTokens) ||
        !make_map(&B.tm_qn12, q_noise, 192, hkv, N, 64, 1, kBwdStepTokens) ||
        !make_map(&B.tm_dhs12, dh_sig, 128, 4 * hkv, N, 64, 4, kBwdStepTokens) ||
        !make_map(&B.tm_dhn12, dh_noise, 128, hkv, N, 64, 1, kBwdStepTokens) ||
        !make_map(&B.tm_k64, k, 192, hkv, N, 64, 1, kBwdQKeyTile) ||
        !make_map(&B.tm_v64, v, 128, hkv, N, 64, 1, kBwdQKeyTile) ||
        !make_map(&B.tm_k128, k, 192, hkv, N, 64, 1, kBwdKeyTile) ||
        !make_map(&B.tm_v128, v, 128, hkv, N, 64, 1, kBwdKeyTile) ||
        !make_map_f32_3d(&B.tm_stats, stats, kBwdStats, hkv, N, kBwdStats, 1, kBwdStepTokens))
        return GDLA_ERR_CUDA;
    B.stats = stats;
    B.dq_sig = static_cast<__nv_bfloat16 *>(dq_sig);
    B.dq_noise = static_cast<__nv_bfloat16 *>(dq_noise);
    B.dk = static_cast<__nv_bfloat16 *>(dk);
    B.dv = static_cast<__nv_bfloat16 *>(dv);
    if (!run_plans(batch, seqlens, hkv, window, T, q_cost(T, kBwdQKeyTile),
                   [&](const PrefillPlan &P) { return launch_bwd_dq(B, P, st) == cudaSuccess; }))
        return GDLA_ERR_CUDA;
    auto kv_cost = [=](int L, int kt) {
        const int u0 = kt * kBwdKeyTile;
        const int t_end = (window > 0) ? std::min(L, u0 + kBwdKeyTile - 1 + window) : L;
        return (t_end - u0 + kBwdStepTokens - 1) / kBwdStepTokens;
    };
    if (!run_plans(batch, seqlens, hkv, window, kBwdKeyTile, kv_cost,
                   [&](const PrefillPlan &P) { return launch_bwd_dkv(B, P, st) == cudaSuccess; }))
        return GDLA_ERR_CUDA;
    return GDLA_OK;
}

size_t gdla_prologue_workspace_bytes(long long total_tokens) {
    if (total_tokens < 0 || total_tokens >= (1ll << 31)) return 0;
    const size_t n = static_cast<size_t>(total_tokens);
    return align256(n * 1024 * 2) + align256(n * 512 * 2) + align256(n * 16 * 4) + align256(n * 64 * 2) +
           align256(n * 64 * 4);
}

gdla_status_t gdla_prologue(const void *x, const void *w_qa, const void *w_kva, const float *gamma_q,
                            const float *gamma_kv, const void *w_qb, const void *w_uk, const void *w_uv,
                            const void *w_lambda, const void *w_gate, void *q_sig, void *q_noise, void *k, void *v,
                            float *lambda, void *gate_logits, int batch, const int32_t *seqlens, int num_kv_heads,
                            void *workspace, size_t workspace_bytes, void *stream) {
    if (batch < 1 || seqlens == nullptr) return GDLA_ERR_INVALID_ARG;
    if (batch > kPrologueMaxSeqs) return GDLA_ERR_UNSUPPORTED;
    if (num_kv_heads < 1 || num_kv_heads > GDLA_MAX_KV_HEADS) return GDLA_ERR_UNSUPPORTED;
    std::unique_ptr<ProloguePlan> plan(new ProloguePlan);
    long long n_total = 0;
    plan->n_seqs = batch;
    for (int b = 0; b < batch; ++b) {
        if (seqlens[b] < 0) return GDLA_ERR_INVALID_ARG;
        plan->starts[b] = static_cast<int>(n_total);
        n_total += seqlens[b];
        if (n_total >= (1ll << 31)) return GDLA_ERR_INVALID_ARG;
    }
    plan->starts[batch] = static_cast<int>(n_total);
    if (n_total == 0) return GDLA_OK;
    const void *bufs[] = {x, w_qa, w_kva, gamma_q, gamma_kv, w_qb, w_uk, w_uv, w_lambda, w_gate,
                          q_sig, q_noise, k, v, lambda, gate_logits};
    for (const void *b : bufs)
        if (!aligned16(b)) return GDLA_ERR_INVALID_ARG;
    const size_t need = gdla_prologue_workspace_bytes(n_total);
    if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return GDLA_ERR_WORKSPACE;
    const int hkv = num_kv_heads;
    const uint64_t N = static_cast<uint64_t>(n_total);
    PrologueLaunch L{};
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    const size_t n = static_cast<size_t>(n_total);
    L.io.cq_g = reinterpret_cast<__nv_bfloat16 *>(w8);
    w8 += align256(n * 1024 * 2);
    L.io.ckv_g = reinterpret_cast<__nv_bfloat16 *>(w8);
    w8 += align256(n * 512 * 2);
    L.io.ssq = reinterpret_cast<float *>(w8);
    w8 += align256(n * 16 * 4);
    L.io.krope = reinterpret_cast<__nv_bfloat16 *>(w8);
    w8 += align256(n * 64 * 2);
    L.io.rot = reinterpret_cast<float *>(w8);
    L.io.gamma_q = gamma_q;
    L.io.gamma_kv = gamma_kv;
    L.io.lambda = lambda;
    L.io.gate = static_cast<__nv_bfloat16 *>(gate_logits);
    L.io.q_sig = static_cast<__nv_bfloat16 *>(q_sig);
    L.io.q_noise = static_cast<__nv_bfloat16 *>(q_noise);
    L.io.k = static_cast<__nv_bfloat16 *>(k);
    L.io.v = static_cast<__nv_bfloat16 *>(v);
    L.io.hkv = hkv;
    // 2-D bf16 operands as [rows][K] maps with 64-wide K boxes (128-byte swizzle); the
    // weights' boxes are half a tile's columns (each CTA of a pair loads one half)
    if (!make_map(&L.tm_x, x, 4096, N, 1, 64, 128, 1) || !make_map(&L.tm_wqa, w_qa, 4096, 1024, 1, 64, 128, 1) ||
        !make_map(&L.tm_wkva, w_kva, 4096, 576, 1, 64, 96, 1) ||
        !make_map(&L.tm_wlam, w_lambda, 4096, 4 * hkv, 1, 64, 32, 1) ||
        !make_map(&L.tm_wgate, w_gate, 4096, 4ull * hkv * 128, 1, 64, 128, 1) ||
        !make_map(&L.tm_cqn, L.io.cq_g, 1024, N, 1, 64, 128, 1) ||
        !make_map(&L.tm_wqb, w_qb, 1024, 5ull * hkv * 192, 1, 64, 128, 1) ||
        !make_map(&L.tm_ckvn, L.io.ckv_g, 512, N, 1, 64, 128, 1) ||
        !make_map(&L.tm_wuk, w_uk, 512, 128ull * hkv, 1, 64, 64, 1) ||
        !make_map(&L.tm_wuv, w_uv, 512, 128ull * hkv, 1, 64, 64, 1) ||
        !make_map(&L.tm_qs_o, q_sig, 192, 4ull * hkv, N, 64, 1, 32) ||
        !make_map(&L.tm_qn_o, q_noise, 192, hkv, N, 64, 1, 32) || !make_map(&L.tm_k_o, k, 192, hkv, N, 64, 1, 32) ||
        !make_map(&L.tm_v_o, v, 128, hkv, N, 64, 1, 32))
        return GDLA_ERR_CUDA;
    if (launch_prologue(L, *plan, static_cast<int>(n_total), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GDLA_ERR_CUDA;
    return GDLA_OK;
}

size_t gdla_decode_workspace_bytes(int batch, int num_kv_heads, int max_seqlen_k, int window) {
    if (batch < 1 || num_kv_heads < 1 || num_kv_heads > GDLA_MAX_KV_HEADS || max_seqlen_k < 1) return 0;
    return decode_workspace_bytes(make_decode_plan(batch, num_kv_heads, max_seqlen_k, window, 1));
}

gdla_status_t gdla_attn_decode(const void *q_sig, const void *q_noise, const void *k_cache, const void *v_cache,
                               const int32_t *cu_seqlens_k, int num_cache_rows, int max_seqlen_k,
                               const float *lambda, const void *gate_logits, void *out, int batch, int num_kv_heads,
                               int window, void *workspace, size_t workspace_bytes, void *stream) {
    if (batch < 1 || num_cache_rows < 1 || max_seqlen_k < 1) return GDLA_ERR_INVALID_ARG;
    if (num_kv_heads < 1 || num_kv_heads > GDLA_MAX_KV_HEADS) return GDLA_ERR_UNSUPPORTED;
    if (!aligned16(q_sig) || !aligned16(q_noise) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(lambda) || !aligned16(gate_logits) || !aligned16(out) || cu_seqlens_k == nullptr ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
        return GDLA_ERR_INVALID_ARG;
    const DecodePlan plan = make_decode_plan(batch, num_kv_heads, max_seqlen_k, window, num_cache_rows);
    const size_t need = decode_workspace_bytes(plan);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                     (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
        return GDLA_ERR_WORKSPACE;
    DecodeLaunch L{};
    const uint64_t nk = static_cast<uint64_t>(num_cache_rows);
    const uint32_t tk = static_cast<uint32_t>(decode_key_tile(plan));
    if (!make_map(&L.tm_k, k_cache, 192, num_kv_heads, nk, 64, 1, tk) ||
        !make_map(&L.tm_v, v_cache, 128, num_kv_heads, nk, 64, 1, tk))
        return GDLA_ERR_CUDA;
    L.q_sig = static_cast<const __nv_bfloat16 *>(q_sig);
    L.q_noise = static_cast<const __nv_bfloat16 *>(q_noise);
    L.cu_seqlens_k = cu_seqlens_k;
    L.lambda = lambda;
    L.gate = static_cast<const __nv_bfloat16 *>(gate_logits);
    L.out = static_cast<__nv_bfloat16 *>(out);
    L.ws = static_cast<float *>(workspace);
    if (launch_decode(L, plan, static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDLA_ERR_CUDA;
    return GDLA_OK;
}

size_t gdla_decode_latent_workspace_bytes(int batch, int num_kv_heads, int max_seqlen_k, int window) {
    if (batch < 1 || num_kv_heads < 1 || num_kv_heads > GDLA_LATENT_MAX_KV_HEADS || max_seqlen_k < 1) return 0;
    return latent_workspace_bytes(make_latent_plan(batch, num_kv_heads, max_seqlen_k, window, 1));
}

gdla_status_t gdla_attn_decode_latent(const void *q_abs_sig, const void *q_abs_noise, const void *ckv,
                                      const int32_t *cu_seqlens_k, int num_cache_rows, int max_seqlen_k,
                                      const void *w_uv, const float *lambda, const void *gate_logits, void *out,
                                      int batch, int num_kv_heads, int window, void *workspace,
                                      size_t workspace_bytes, void *stream) {
    if (batch < 1 || num_cache_rows < 1 || max_seqlen_k < 1) return GDLA_ERR_INVALID_ARG;
    if (num_kv_heads < 1 || num_kv_heads > GDLA_LATENT_MAX_KV_HEADS) return GDLA_ERR_UNSUPPORTED;
    if (!aligned16(q_abs_sig) || !aligned16(q_abs_noise) || !aligned16(ckv) || !aligned16(w_uv) ||
        !aligned16(lambda) || !aligned16(gate_logits) || !aligned16(out) || cu_seqlens_k == nullptr ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
        return GDLA_ERR_INVALID_ARG;
    const LatentPlan plan = make_latent_plan(batch, num_kv_heads, max_seqlen_k, window, num_cache_rows);
    const size_t need = latent_workspace_bytes(plan);
    if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return GDLA_ERR_WORKSPACE;
    LatentLaunch L{};
    const int hkv = num_kv_heads;
    // Q boxes: one sequence's 4H signal rows and H noise rows, 64 dims at a time;
    // latent cache: 48 rows x 64 dims; W^UV_j: its 128 rows x 64 dims.
    if (!make_map(&L.tm_qs, q_abs_sig, 576, 4 * hkv, static_cast<uint64_t>(batch), 64, 4 * hkv, 1) ||
        !make_map(&L.tm_qn, q_abs_noise, 576, hkv, static_cast<uint64_t>(batch), 64, hkv, 1) ||
        !make_map(&L.tm_c, ckv, 576, 1, static_cast<uint64_t>(num_cache_rows), 64, 1, 48) ||
        !make_map(&L.tm_w, w_uv, 512, 128, static_cast<uint64_t>(hkv), 64, 128, 1))
        return GDLA_ERR_CUDA;
    L.cu_seqlens_k = cu_seqlens_k;
    L.lambda = lambda;
    L.gate = static_cast<const __nv_bfloat16 *>(gate_logits);
    L.out = static_cast<__nv_bfloat16 *>(out);
    L.ws = static_cast<float *>(workspace);
    if (launch_decode_latent(L, plan, static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDLA_ERR_CUDA;
    return GDLA_OK;
}

int gdla_device_error(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

const char *gdla_status_string(gdla_status_t status) {
    switch (status) {
        case GDLA_OK: return "GDLA_OK";
        case GDLA_ERR_INVALID_ARG: return "GDLA_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
        case GDLA_ERR_UNSUPPORTED: return "GDLA_ERR_UNSUPPORTED: sizes outside what the kernels handle";
        case GDLA_ERR_WORKSPACE: return "GDLA_ERR_WORKSPACE: decode workspace missing, misaligned or too small";
        case GDLA_ERR_CUDA: return "GDLA_ERR_CUDA: a CUDA call or kernel launch failed";
    }
    return "GDLA: unknown status";
}

int gdla_version(void) { return GDLA_VERSION; }

}  // extern "C"
