// gdla_internal.h - launch plans shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace gdla {

// Prefill: one MMA tile = 24 tokens x 5 heads = 120 of the 128 MMA rows. The
// CTA size and key tile depend on the window (see prefill_geometry).
constexpr int kPrefillTileTokens = 24;
constexpr int kPrefillSlidingMaxWindow = 256;  // windows up to this use the sliding configuration

struct PrefillGeometry {
    int cta_tokens;       // tokens per CTA (a multiple of kPrefillTileTokens)
    int key_tile;         // keys per K/V tile
    int v_box;            // keys per V TMA box
    bool async_epilogue;  // gate/lambda/output tensor maps are used
};
PrefillGeometry prefill_geometry(int window);
constexpr int kPlanMaxSeqs = 256;    // sequences per launch (more are split across launches)
constexpr int kPlanMaxItems = 6144;  // q-tiles per launch
constexpr int kItemSeqShift = 20;
constexpr uint32_t kItemTileMask = (1u << kItemSeqShift) - 1u;

// Work item of a persistent CTA in its round r (0, 1, ...): the CTAs take the
// list round-robin, in reverse order on odd rounds, so that over a list sorted
// heaviest first every CTA gets a similar total (plain round-robin hands CTA 0
// the heaviest item of every round).
__device__ __forceinline__ int snake_item(int r) {
    const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return r * g + ((r & 1) ? g - 1 - c : c);
}

// Passed by value (kernel parameters): the q-tiles of one launch, heaviest
// first. The host builds the largest form and launches the smallest capacity
// that holds the plan, so a launch carries ~3.3 KB, ~8.7 KB or ~26.6 KB.
template <int MAX_ITEMS, int MAX_SEQS>
struct PrefillPlanT {
    static constexpr int kMaxItems = MAX_ITEMS;
    static constexpr int kMaxSeqs = MAX_SEQS;
    int n_items;
    int hkv;
    int window;
    int n_seqs;
    int seq_start[MAX_SEQS];  // packed row of each sequence's first token
    int seq_len[MAX_SEQS];
    uint32_t items[MAX_ITEMS];  // (local sequence << kItemSeqShift) | CTA block index
};
using PrefillPlan = PrefillPlanT<kPlanMaxItems, kPlanMaxSeqs>;
using PrefillPlanMedium = PrefillPlanT<2048, 64>;
using PrefillPlanSmall = PrefillPlanT<768, 32>;

// Backward: what the forward recompute leaves for the gradient kernels (and the
// gradients it finishes itself). Row statistics per (token, KV group): the
// base-2 log-sum-exp of the scaled scores of heads 0..4 (4 signal, noise) at
// 0..4, and rowsum(dH * H) of the same heads at 8..12.
constexpr int kBwdStats = 16;
struct BwdIO {
    const __nv_bfloat16 *dout;   // [N, 4H, 128]
    __nv_bfloat16 *dgate;        // [N, 4H, 128]
    float *dlambda;              // [N, 4H]
    __nv_bfloat16 *dh_sig;       // [N, 4H, 128]: gradient of H_S (= dout * sigmoid(gate)), bf16
    __nv_bfloat16 *dh_noise;     // [N, H, 128]: gradient of H_N, bf16
    float *stats;                // [N, H, kBwdStats]
};

struct PrefillLaunch {
    CUtensorMap tm_qs, tm_qn, tm_k, tm_v;
    CUtensorMap tm_gate, tm_lam, tm_out;  // used by the asynchronous epilogue (short windows)
    const float *lambda;
    const __nv_bfloat16 *gate;
    __nv_bfloat16 *out;
    BwdIO bwd;                            // backward recompute only
};

// Backward gradient kernels (gdla_prefill_bwd.cu). Plans: dq - items are 24-token
// q tiles (cost: 64-key tiles visited); dkv - items are 128-key tiles (cost:
// 12-token steps over the rows that see them).
constexpr int kBwdQKeyTile = 64;
constexpr int kBwdKeyTile = 128;
constexpr int kBwdStepTokens = 12;
struct BwdLaunch {
    CUtensorMap tm_qs, tm_qn;       // Q boxes of 6 tokens (as the forward)
    CUtensorMap tm_dhs, tm_dhn;     // dH boxes of 6 tokens
    CUtensorMap tm_qs12, tm_qn12;   // Q boxes of 12 tokens (dkv steps)
    CUtensorMap tm_dhs12, tm_dhn12; // dH boxes of 12 tokens
    CUtensorMap tm_k64, tm_v64;     // 64-key K / V boxes (dq)
    CUtensorMap tm_k128, tm_v128;   // 128-key K / V boxes (dkv)
    CUtensorMap tm_stats;           // row statistics, 12 tokens of one group
    const float *stats;
    __nv_bfloat16 *dq_sig, *dq_noise, *dk, *dv;
};
cudaError_t launch_bwd_dq(const BwdLaunch &launch, const PrefillPlan &plan, cudaStream_t stream);
cudaError_t launch_bwd_dkv(const BwdLaunch &launch, const PrefillPlan &plan, cudaStream_t stream);

cudaError_t launch_prefill(const PrefillLaunch &launch, const PrefillPlan &plan, cudaStream_t stream);
// Backward, first pass: the forward recomputed on the forward's schedule for the
// plan's window (prefill_geometry), writing launch.bwd instead of the output.
cudaError_t launch_prefill_bwd_recompute(const PrefillLaunch &launch, const PrefillPlan &plan, cudaStream_t stream);

// SM count of a device, queried once per device and cached (0 on failure).
constexpr int kMaxCachedDevices = 64;
int device_sm_count(int dev);

// Identifier of the CUDA context current on the calling thread (0 if none is
// current or it cannot be read). Tearing the primary context down (a device
// reset) and re-creating it gives a new identifier, so host caches of facts
// that belong to a context (kernel attribute opt-ins, symbol addresses) key
// on it and are refreshed after a reset.
unsigned long long current_context_id();

// One flag per device, valid for one context: set() records the context it was
// set in, is_set() holds only while that context is still the current one.
struct PerContextFlag {
    std::atomic<unsigned long long> ctx[kMaxCachedDevices];
    bool is_set(int dev, unsigned long long id) const {
        return id != 0 && dev >= 0 && dev < kMaxCachedDevices && ctx[dev].load(std::memory_order_relaxed) == id;
    }
    void set(int dev, unsigned long long id) {
        if (id != 0 && dev >= 0 && dev < kMaxCachedDevices) ctx[dev].store(id, std::memory_order_relaxed);
    }
};

// Decode: split-KV.
constexpr int kDecodeMaxSplits = 64;
constexpr int kDecodeMinSplitKeys = 1024;

struct DecodePlan {
    int batch;
    int hkv;
    int window;
    int max_seqlen_k;
    int num_cache_rows;
    int num_splits;
    int split_keys;        // keys per split (multiple of 64)
    long long ml_offset_floats;  // start of the (m, l) area in the workspace, in floats
};

struct DecodeLaunch {
    CUtensorMap tm_k, tm_v;
    const __nv_bfloat16 *q_sig, *q_noise;
    const int32_t *cu_seqlens_k;
    const float *lambda;
    const __nv_bfloat16 *gate;
    __nv_bfloat16 *out;
    float *ws;
};

cudaError_t launch_decode(const DecodeLaunch &launch, const DecodePlan &plan, cudaStream_t stream);
int decode_smem_bytes();

// Decode over the latent cache: split-KV, then a combine with the W^UV up-projection.
constexpr int kLatentMaxSplits = 32;
constexpr int kLatentMinSplitKeys = 2048;

struct LatentPlan {
    int batch;
    int hkv;
    int window;
    int max_seqlen_k;
    int num_cache_rows;
    int num_splits;
    int split_keys;              // keys per split (multiple of the 48-key stage)
    long long ml_offset_floats;  // start of the (m, l) area in the workspace, in floats
};

struct LatentLaunch {
    CUtensorMap tm_qs, tm_qn, tm_c, tm_w;
    const int32_t *cu_seqlens_k;
    const float *lambda;
    const __nv_bfloat16 *gate;
    __nv_bfloat16 *out;
    float *ws;
};

LatentPlan make_latent_plan(int batch, int hkv, int max_seqlen_k, int window, int num_cache_rows);
size_t latent_workspace_bytes(const LatentPlan &plan);
cudaError_t launch_decode_latent(const LatentLaunch &launch, const LatentPlan &plan, cudaStream_t stream);

// Host-side decode split plan (shared by the workspace query and the launch).
DecodePlan make_decode_plan(int batch, int hkv, int max_seqlen_k, int window, int num_cache_rows);
size_t decode_workspace_bytes(const DecodePlan &plan);

}  // namespace gdla
