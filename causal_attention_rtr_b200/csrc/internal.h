// internal.h -- declarations shared by the host side of librtr and its
// kernels (not part of the public C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <vector>

#include "rtr.h"

namespace rtr {

// One contiguous run of keys the query rows attend to.
//   src 0: head-major source [heads][rows][d] (KV cache, text cache)
//   src 1: token-major source [rows][heads][d] (current chunk, prefill
//          sequence)
//   causal: key j of the run (0-based) is visible to query row i (0-based)
//          iff floor(j / kpf) <= floor(i / kpf); the run and the query rows
//          start on the same frame boundary.  Otherwise every key is visible.
struct KvSeg {
    int src;
    int row0;
    int len;
    int causal;
};

constexpr int kMaxSegs = 4;

// Work description shared by the tensor-core and the fp32 attention kernels.
struct AttnProblem {
    int nq;          // query rows (token-major [nq][heads][d])
    int heads;
    int head_dim;
    int kpf;         // tokens per latent frame for causal runs
    int nseg;
    KvSeg seg[kMaxSegs];
    float scale;     // multiplies q.k
    // raw pointers (fp32 path) / bases for the tensor maps (bf16 path)
    const void *q;
    void *o;
    const void *k0, *v0;   // head-major source
    long long rows0;       // rows per head of the head-major source
    const void *k1, *v1;   // token-major source
    long long rows1;       // rows of the token-major source
    // Optional write of the token-major source (the chunk) into the
    // head-major buffers commit_k / commit_v ([heads][rows0][d]) by the same
    // launch: row r of chunk frame c = r / kpf goes to row commit_row0 +
    // ((commit_first_slot + c) mod commit_slots) * kpf + r mod kpf.  Null
    // commit_k: no write.  The rows written must be disjoint from every key
    // run the launch reads.
    void *commit_k, *commit_v;
    int commit_first_slot, commit_slots, commit_row0;
    // Optional device array of tensor maps, [commit_slots][K, V][128-row box,
    // 8-row box], each over one ring slot's k rows (128-byte swizzle): the
    // chunk write is then a few TMA stores issued by one thread.  Null: the
    // chunk-write warps copy rows themselves.
    const CUtensorMap *commit_maps;
    // Optional row statistics: lse[h * nq + i] = log sum_j exp(scale q_i.k_j)
    // over the keys row i sees (natural log, fp32).  Null: not written.
    float *lse;
    // Optional fp32 output (bf16 path, one CTA per MMA, no chunk write):
    // token-major [nq][heads][d] written instead of the bf16 `o`.
    float *o_f32;
};

// Schedule of the persistent tensor-core kernel for one problem: units are
// (head, 256-row query pair); full rounds give every CTA one whole unit, the
// remaining units' key tiles are cut into per-CTA ranges that even out the
// CTAs' totals.
struct AttnPlan {
    int cg;                    // CTAs per cluster sharing each MMA (1, or 2 for the CTA pair)
    int unit_rows;             // query rows per unit: 256 per CTA of the cluster
    int n_pairs, n_units, grid, full_rounds, head_major;   // grid: clusters
    std::vector<int> rem_lo;   // grid + 1 boundaries of the per-CTA remainder ranges
    std::vector<int> rem_U;    // key-tile offset of each remainder unit
    bool has_split;            // some unit is shared by two CTAs (combine kernel runs)
    size_t scratch_bytes;      // partial results of split units
};

void plan_attn_bf16(const AttnProblem &p, int sms, int cg, AttnPlan &plan);

// Backward pass of the block-causal attention over one sequence (bf16).
// Token-major [n][heads][head_dim] tensors; lse [heads][n] natural-log row
// log-sum-exp from the forward.
struct BwdProblem {
    const void *q, *k, *v, *o, *dout;
    const float *lse;
    void *dq, *dk, *dv;
    int n, heads, head_dim, kpf;
    float scale;
};
size_t bwd_scratch_bytes(int n, int heads);
cudaError_t launch_attn_bwd(const BwdProblem &p, unsigned *status, void *scratch, cudaStream_t s);

// Argument checks and defaults shared by every entry point.
bool shape_ok(int heads, int head_dim);                 // heads >= 1, head_dim 64 or 128
float resolve_scale(float scale, int head_dim);         // scale > 0 ? scale : 1 / sqrt(head_dim)
int sm_count(int device);                               // SMs of `device` (cached; 148 if unknown)

// Kernel launchers; return cudaSuccess or the launch error.
cudaError_t launch_attn_bf16(const AttnProblem &p, const AttnPlan &plan, const CUtensorMap *tm_k0,
                             const CUtensorMap *tm_k0h, const CUtensorMap *tm_v0, unsigned *status, void *scratch,
                             cudaStream_t s);
cudaError_t launch_attn_f32(const AttnProblem &p, cudaStream_t s);

// Copy n_tok rows of [n_tok][heads][d] into a head-major buffer
// [heads][rows_per_head][d]: token t of frame f = t / k_frame goes to row
// ((first_slot + f) mod slot_mod + slot_off) * k_frame + t mod k_frame.
// K and V move in one launch.
struct ScatterArgs {
    const void *src_k, *src_v;
    void *dst_k, *dst_v;
    int n_tok, heads, row_bytes, k_frame;
    int first_slot, slot_mod, slot_off;
    long long rows_per_head;
};
cudaError_t launch_kv_scatter(const ScatterArgs &a, cudaStream_t s);

// Tensor map for a 3-D tensor of bf16 [outer][mid][d] with a box of
// (64, box_mid, box_outer) elements and 128-byte swizzle.
bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t d, uint64_t mid, uint64_t outer,
                    uint32_t box_mid, uint32_t box_outer);
// The same with an explicit byte stride between `outer` entries.
bool make_tmap_bf16_strided(CUtensorMap *m, const void *base, uint64_t d, uint64_t mid, uint64_t outer,
                            uint64_t stride_outer, uint32_t box_mid, uint32_t box_outer);

unsigned *device_status_ptr(int device);

// Count of kernels this library has launched (all devices, since load).
void count_launch(int n = 1);

// Test hook: the next `launches` tensor-core attention launches on `device`
// issue no loads, so their bounded waits expire and latch RTR_E_TIMEOUT.
void inject_wait_timeouts(int device, int launches);

}  // namespace rtr
