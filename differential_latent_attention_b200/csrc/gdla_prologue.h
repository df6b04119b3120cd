// gdla_prologue.h - launch description of the prologue projections (gdla_prologue.cu),
// shared with the C-ABI layer.
#pragma once

#include "gdla_internal.h"

namespace gdla {

// Error-site tag of the prologue kernels' bounded waits (beside the ERR_SITE_* of gdla_ptx.cuh).
constexpr int ERR_SITE_PROLOGUE = 16 << 16;

constexpr int kPrologueMaxSeqs = 1024;
struct ProloguePlan {
    int n_seqs;
    int starts[kPrologueMaxSeqs + 1];  // packed row of each sequence's first token; starts[n_seqs] = N
};
struct PrologueIO {
    __nv_bfloat16 *cq_g, *ckv_g;      // workspace: c^Q * gamma_q [N, 1024], c^KV * gamma_kv [N, 512] (bf16)
    float *ssq;                       // workspace: [N, 16] partial sums of squares (0-7 of c^Q, 8-13 of c^KV)
    __nv_bfloat16 *krope;             // workspace: rotated k^R [N, 64]
    float *rot;                       // workspace: [N, 64] cos (0..31), sin (32..63) of each row's angles
    const float *gamma_q, *gamma_kv;  // RMSNorm weights [1024], [512]
    float *lambda;                    // out: [N, 4H]
    __nv_bfloat16 *gate;              // out: [N, 4H, 128]
    __nv_bfloat16 *q_sig, *q_noise, *k, *v;  // out
    int hkv;
};
// One GEMM problem of a grouped projection launch: its tiles are 256 rows (a CTA
// pair) x nt columns over K = 64 nk, numbered from `first` with the row block fastest.
struct ProjProblem {
    int epi, nt, nk, n_tiles, first;
};
constexpr int kProjMaxProblems = 4;
struct ProjGroup {
    CUtensorMap tm_a[kProjMaxProblems], tm_b[kProjMaxProblems];
    CUtensorMap tm_o[4];  // TMA store targets of the up-projections: q_sig, q_noise, k, v (64-dim x 32-row boxes)
    ProjProblem prob[kProjMaxProblems];
    int n_prob, m_pairs, total_tiles, M;  // m_pairs: 256-row blocks
};
struct PrologueLaunch {
    CUtensorMap tm_x, tm_wqa, tm_wkva, tm_wlam, tm_wgate;  // projections of x (K = 4096)
    CUtensorMap tm_cqn, tm_wqb;                            // query up-projection (K = 1024)
    CUtensorMap tm_ckvn, tm_wuk, tm_wuv;                   // KV up-projection (K = 512)
    CUtensorMap tm_qs_o, tm_qn_o, tm_k_o, tm_v_o;          // up-projection outputs (store boxes)
    PrologueIO io;
};
cudaError_t launch_prologue(const PrologueLaunch &launch, const ProloguePlan &plan, int total_tokens,
                            cudaStream_t stream);


}  // namespace gdla
