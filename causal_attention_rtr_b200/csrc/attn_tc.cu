// attn_tc.cu -- frame-causal flash-attention forward for B200 (sm_100a) on the
// 5th-generation tensor cores.
//
// Computes, per head, O = softmax(Q K^T * scale + M) V where M is the
// temporal causal mask of RTR-DiT (papernotes.org note "DiT as Real-Time
// Rerenderer", Method > Key Designs 2: a query in latent frame floor(i/k) sees
// keys of frames floor(j/k) <= floor(i/k)).  Keys arrive as up to four
// contiguous runs (KvSeg): the anchored reference and the ring-buffer window
// of the KV cache (always visible to the chunk; Key Designs 4), and the chunk
// itself or a whole sequence (frame-causal).  The mask is resolved at tile
// granularity: key tiles past the last visible frame of a query-tile pair are
// never loaded, fully visible tiles take no mask work, and only tiles that
// straddle a frame boundary or a run's end mask element-wise.
//
// Work unit: one head x 256 query rows (two 128-row tiles Q0, Q1 sharing one
// K/V stream).  The kernel is persistent, one CTA per SM.  Units are ordered
// largest first; CTA c takes units c, c+G, c+2G, ... for as many full rounds as
// there are units for every CTA, then an equal share of the remaining units'
// key tiles.  A unit split across CTAs writes an unnormalised fp32 partial
// (O, running max, row sum) to scratch and attn_combine merges the parts.
// Full rounds start every CTA at key tile 0 of a unit, so CTAs that work on
// the same head sweep its cache together and share it through L2.
//
// One CTA, 384 threads:
//   warp 0      TMA producer: Q0/Q1 per unit, then K_j, V_j into a 4-slot ring
//   warp 1      tcgen05 issuer (one thread): S_i = Q_i K_j^T into TMEM,
//               O_i += P_i V_j with P_i read from TMEM (the "A in tensor
//               memory" form), commits to mbarriers
//   warps 2-3   chunk write (rtr_attn_frame_causal_commit): copy the chunk's
//               key / value tiles from the ring slots to their cache rows;
//               idle otherwise
//   warps 4-7   softmax for Q0, warps 8-11 softmax for Q1: one thread per
//               query row reads its 128 scores from TMEM once into registers,
//               online softmax in fp32 (exp2 domain; O is rescaled only when
//               the running max grows by more than 2^8 -- exact after the
//               final division), writes P as bf16 back over its S columns in
//               four 32-key chunks, and finally normalises O and stores it
//               with TMA (or writes the fp32 partial).  Once P of the first
//               64 keys is stored the tensor core starts their half of PV,
//               while the softmax finishes the other half.
// The two softmax groups ping-pong: while one works on its S tile the tensor
// core runs the other tile's QK^T or PV.  Part of the exponentials run as a
// polynomial on the FMA pipe (exp2_poly) so that the special-function unit
// is not the bottleneck.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// Shared memory: Q0, Q1 and 4 K/V slots, each 128 rows x D bf16 stored as D/64
// boxes of 128 rows x 128 bytes with the 128-byte swizzle that TMA writes and
// the tcgen05 descriptors read.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "exp2_poly.h"
#include "internal.h"
#include "ptx.cuh"

#ifndef RTR_REGS_LOW
#define RTR_REGS_LOW 120     // producer / MMA warpgroup after setmaxnreg
#endif
#define RTR_REGS_HIGH (168 + (168 - RTR_REGS_LOW) / 2)   // each softmax warpgroup
#ifndef RTR_UNIT_ORDER_RATIO
#define RTR_UNIT_ORDER_RATIO 1.25   // head-major unit order when max/min key tiles per pair <= this
#endif
#ifndef RTR_PV_SPLIT
#define RTR_PV_SPLIT 1   // PV over the first 64 keys starts once their P is stored (bPh); 0: after all of P
#endif
#ifndef RTR_SOFTMAX_1LD
#define RTR_SOFTMAX_1LD 1   // the row's 128 scores read from TMEM once, held in registers; 0: read twice
#endif
#ifndef RTR_EXP2_POLY_PER8
#define RTR_EXP2_POLY_PER8 0   // of every 8 scores, how many use exp2_poly (0 measured fastest so far)
#endif

namespace rtr {

__device__ unsigned g_device_status;   // RTR_OK or RTR_E_TIMEOUT, latched

namespace {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kPairRows = 2 * kBM;   // query rows per CTA (two tiles)
constexpr int kThreads = 384;     // 12 warps
constexpr int kMaxGrid = 160;     // persistent CTAs at most (B200: 148 SMs)
constexpr uint64_t kWaitNs = 1000000000ull;   // bounded waits: 1 s
constexpr long long kSplitPenaltyTiles = 15;   // a split unit's extra cost, in key-tile steps (planner)

struct TcParams {
    CUtensorMap tm_q;   // token-major [nq][H][D], box (64, 1, 128)
    CUtensorMap tm_o;   // token-major output
    CUtensorMap tm_k0;  // head-major [H][rows][D], box (64, 128, 1)
    CUtensorMap tm_v0;
    CUtensorMap tm_k1;  // token-major [rows][H][D], box (64, 1, 128)
    CUtensorMap tm_v1;
    CUtensorMap tm_k0h; // K maps with 64-row boxes (CTA-pair mode: each CTA loads half a key tile)
    CUtensorMap tm_k1h;
    int nq, heads, kpf, nseg;
    int unit_rows;      // query rows per work unit: 256 per CTA of the cluster
    KvSeg seg[kMaxSegs];
    float scale_log2;   // scale * log2(e)
    unsigned *status;
    int test_skip_loads;   // test hook: issue no loads, so the bounded waits expire
    // schedule: full rounds, then CTA c takes tiles [rem_lo[c], rem_lo[c+1])
    // of the remaining units' key tiles
    int n_pairs, n_units, grid, full_rounds, head_major;   // n_pairs: row blocks of unit_rows per head; grid: clusters
    int rem_lo[kMaxGrid + 1];
    int rem_U[kMaxGrid];   // key tiles of the remainder before its unit i (fewer than kMaxGrid units)
    float4 *part_o;     // [CTAs][2][D/4][256]
    float2 *part_ml;    // [CTAs][2][256]: running max (log2 units), row sum
    __nv_bfloat16 *out; // token-major output (combine kernel)
    // chunk write: the src-1 run's rows into the ring of the head-major
    // buffers (null commit_k: none); see AttnProblem
    __nv_bfloat16 *commit_k, *commit_v;
    long long commit_rows_per_head;
    int commit_first_slot, commit_slots, commit_row0;
    const CUtensorMap *commit_maps;   // per-slot store maps (see AttnProblem) or null
    float *lse;         // [heads][nq] natural-log row log-sum-exp, or null
    float *out_f32;     // token-major fp32 output instead of bf16 (whole rows stored directly), or null
};

// CG = CTAs per cluster working one MMA: 1, or 2 for the CTA-pair MMA
// (tcgen05 cta_group::2: M = 256 rows across the pair, each CTA holding half
// of every key / value tile).
template <int D, int CG>
struct Layout {
    static constexpr int kTileBytes = kBM * D * 2;          // one Q / K / V tile
    static constexpr int kSlotBytes = kTileBytes / CG;      // this CTA's part of a K or V tile
    static constexpr int kSlots = 4 * CG;                   // ring: 128 KB of K/V in flight
    static constexpr int kQ = 0;                            // Q0, Q1
    static constexpr int kKV = 2 * kTileBytes;              // ring slots
    static constexpr int kBars = kKV + kSlots * kSlotBytes; // mbarriers
    static constexpr int bQ = 0, bQfree = 1, bFull = 2, bEmpty = bFull + kSlots, bCopied = bEmpty + kSlots,
                         bGo = bCopied + kSlots, bS = bGo + kSlots, bP = bS + 2, bO = bP + 2, bEpi = bO + 2, bDrain = bEpi + 2,
                         bPh = bDrain + 1, kNumBars = bPh + 2;
    static constexpr int kMisc = kBars + kNumBars * 8;      // tmem holder, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;            // slack for 1 KB alignment
};

// Key tiles of one run for the unit whose rows start at q0.
__device__ __forceinline__ int seg_tiles(const TcParams &p, int s, int q0) {
    const KvSeg &g = p.seg[s];
    int len = g.len;
    if (g.causal) {
        const int q_last = min(q0 + p.unit_rows - 1, p.nq - 1);
        const int lim = (q_last / p.kpf + 1) * p.kpf;
        len = len < lim ? len : lim;
    }
    return (len + kBN - 1) / kBN;
}

__device__ __forceinline__ int pair_tiles(const TcParams &p, int pair) {
    int t = 0;
    for (int s = 0; s < p.nseg; ++s) t += seg_tiles(p, s, pair * p.unit_rows);
    return t;
}

// Unit u -> (pair, head).  Pairs of similar size: head-major (a head's pairs
// are consecutive units, so a full round sweeps whole heads together and the
// shared remainder covers few heads); very unequal pairs (block-causal
// prefill): largest pairs first across heads, so a round's units are alike.
__device__ __forceinline__ void unit_coords(const TcParams &p, int u, int &pair, int &head) {
    if (p.head_major) {
        head = u / p.n_pairs;
        pair = p.n_pairs - 1 - u % p.n_pairs;
    } else {
        pair = p.n_pairs - 1 - u / p.heads;
        head = u % p.heads;
    }
}

// Unit of CTA c in full round r: rounds alternate direction so that CTAs that
// get a larger unit in one round get a smaller one in the next.
__host__ __device__ __forceinline__ int full_round_unit(int G, int c, int r) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

struct Item {
    int unit, t0, t1, slot;   // slot -1: whole unit (final output); 0/1: partial
    int T;                    // key tiles of the whole unit
};

// Deterministic per-CTA work sequence; every role walks the same sequence.
struct Sched {
    int r = 0, ru = 0;
    long long U = 0;
    bool first_rem = true;
    bool placed = false;   // remainder walk moved to this CTA's first unit
};

template <int CG>
__device__ bool sched_next(const TcParams &p, Sched &s, Item &it) {
    const int c = blockIdx.x / CG;   // cluster
    if (s.r < p.full_rounds) {
        it.unit = full_round_unit(p.grid, c, s.r);
        int pair, head;
        unit_coords(p, it.unit, pair, head);
        it.T = pair_tiles(p, pair);
        it.t0 = 0;
        it.t1 = it.T;
        it.slot = -1;
        ++s.r;
        if (s.r == p.full_rounds) s.ru = p.full_rounds * p.grid;
        return true;
    }
    const long long lo = p.rem_lo[c];
    const long long hi = p.rem_lo[c + 1];
    if (!s.placed) {
        // Jump to the last remainder unit that starts at or before this CTA's
        // first tile (binary search of the tile prefix): the units before it
        // end at or before `lo`.  Walking them one by one cost a few hundred
        // cycles each, tens of microseconds for the last CTAs of a launch.
        s.placed = true;
        const int base = s.ru;
        int a = 0, b = p.n_units - base;   // rem_U[a] <= lo; answer in [a, b)
        if (b > 0) {
            while (b - a > 1) {
                const int m = (a + b) >> 1;
                if (p.rem_U[m] <= lo) a = m; else b = m;
            }
            s.ru = base + a;
            s.U = p.rem_U[a];
        }
    }
    while (s.ru < p.n_units && s.U < hi) {
        int pair, head;
        unit_coords(p, s.ru, pair, head);
        const int T = pair_tiles(p, pair);
        const long long a = max(s.U, lo), b = min(s.U + T, hi);
        const int u = s.ru;
        const long long U0 = s.U;
        ++s.ru;
        s.U += T;
        if (a < b) {
            it.unit = u;
            it.T = T;
            it.t0 = (int)(a - U0);
            it.t1 = (int)(b - U0);
            it.slot = (it.t0 == 0 && it.t1 == T) ? -1 : (s.first_rem ? 0 : 1);
            s.first_rem = false;
            return true;
        }
    }
    return false;
}

__device__ __forceinline__ void raise_timeout(const TcParams &p, volatile int *abort_flag) {
    *abort_flag = 1;
    atomicExch(p.status, (unsigned)RTR_E_TIMEOUT);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <uint32_t N>
__device__ __forceinline__ void set_max_regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N>
__device__ __forceinline__ void set_max_regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// Walk the key runs to the run holding unit tile t: returns the run and the
// tile's index within it.
__device__ __forceinline__ void locate_tile(const TcParams &p, int q0, int t, int &s, int &tt) {
    s = 0;
    while (s < p.nseg - 1) {
        const int n = seg_tiles(p, s, q0);
        if (t < n) break;
        t -= n;
        ++s;
    }
    tt = t;
}

// P = exp2(s * scale_log2 - m) for 32 scores of a row, packed to 16 bf16
// pairs and stored at TMEM column `tP`; row sums into acc.  The scale-and-
// shift and the sums use packed f32x2 instructions.
template <bool POLY>
__device__ __forceinline__ void softmax_chunk(const uint32_t (&sr)[32], float sl2, float neg_m, uint32_t tP,
                                              float2 (&acc)[4]) {
    const float2 sl2x2 = make_float2(sl2, sl2), negm2 = make_float2(neg_m, neg_m);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 x = ffma2(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sl2x2, negm2);
        const bool poly = POLY && (e % 4) < (RTR_EXP2_POLY_PER8 / 2);
        const float2 pr = poly ? exp2_poly_x2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
        acc[e & 3] = fadd2(acc[e & 3], pr);
        pk[e] = pack_bf16x2(pr.x, pr.y);
    }
    tmem_st16(tP, pk);
}

// softmax_chunk on 32 scores held at sr[0..31] of a register-resident row.
template <bool POLY>
__device__ __forceinline__ void softmax_chunk_regs(const uint32_t *sr, float sl2, float neg_m, uint32_t tP,
                                                   float2 (&acc)[4]) {
    const float2 sl2x2 = make_float2(sl2, sl2), negm2 = make_float2(neg_m, neg_m);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 x = ffma2(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sl2x2, negm2);
        const bool poly = POLY && (e % 4) < (RTR_EXP2_POLY_PER8 / 2);
        const float2 pr = poly ? exp2_poly_x2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
        acc[e & 3] = fadd2(acc[e & 3], pr);
        pk[e] = pack_bf16x2(pr.x, pr.y);
    }
    tmem_st16(tP, pk);
}

// Chunk write: rows [64*part, 64*part+64) of chunk key (or value) tile tt,
// held in shared memory at `src` in the TMA layout (D/64 boxes of 128 rows x
// 128 bytes, 128-byte swizzle), stored to their ring rows.  Lanes cover
// consecutive 16-byte pieces of a row, so each row is one contiguous store.
template <int D>
__device__ __forceinline__ void commit_tile_rows(const TcParams &p, uint32_t src, __nv_bfloat16 *dst, int head,
                                                 int tt, int part, int lane) {
    constexpr int kPieces = D / 8;          // 16-byte pieces per row
    constexpr int kRowsPerStep = 32 / kPieces;
    const int piece = lane % kPieces, sub = lane / kPieces;
    const int box = piece / 8, c16 = piece % 8;
    // Ring row of chunk row r in frame f: commit_row0 + slot(f) * kpf + r - f * kpf.
    auto ring_row = [&](int r, int f) {
        int slot = p.commit_first_slot + f;           // < 2 * commit_slots
        if (slot >= p.commit_slots) slot -= p.commit_slots;
        return p.commit_row0 + (long long)slot * p.kpf + (r - f * p.kpf);
    };
    const int rbase = tt * kBN + 64 * part;
    const int f0 = rbase / p.kpf;                     // frame of the first row
    const int r_next = (f0 + 1) * p.kpf;              // first row of the next frame
    const long long off0 = ring_row(rbase, f0) - rbase;
#pragma unroll 4
    for (int r0 = 0; r0 < 64; r0 += kRowsPerStep) {
        const int row = 64 * part + r0 + sub;         // row within the tile
        const int r = tt * kBN + row;                 // chunk row
        if (r < p.nq) {
            const long long drow = r < r_next ? off0 + r : ring_row(r, r / p.kpf);
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(src + box * 16384 + row * 128 + ((c16 ^ (row & 7)) << 4)));
            *reinterpret_cast<uint4 *>(dst + ((long long)head * p.commit_rows_per_head + drow) * D + piece * 8) = v;
        }
    }
}

// Chunk write by TMA: the 128 rows of chunk key (or value) tile tt, held in
// shared memory at `src` in the TMA layout, stored to their ring slots by one
// thread.  A tile inside one frame is one 128-row box per 64 columns; the
// pieces of a tile that straddles frames (or ends the chunk) go out as 8-row
// boxes, all starting on a 1024-byte swizzle atom (frame boundaries are
// multiples of 8 rows).  Returns after the stores have read shared memory.
template <int D>
__device__ __forceinline__ void commit_tile_tma(const TcParams &p, uint32_t src, int kv, int head, int tt) {
    const int r0 = tt * kBN, r_end = min(r0 + kBN, p.nq);
    fence_proxy_async_smem();
    for (int r = r0; r < r_end;) {
        const int f = r / p.kpf;
        const int seg_end = min(r_end, (f + 1) * p.kpf);
        int slot = p.commit_first_slot + f;               // < 2 * commit_slots
        if (slot >= p.commit_slots) slot -= p.commit_slots;
        const CUtensorMap *m128 = p.commit_maps + (slot * 2 + kv) * 2;
        const int y = r - f * p.kpf, a = r - r0, len = seg_end - r;
        if (a == 0 && len == kBN) {
#pragma unroll
            for (int b = 0; b < D / 64; ++b) tma_store_3d(m128, src + b * 16384, b * 64, y, head);
        } else {
            for (int i = 0; i < len; i += 8)
#pragma unroll
                for (int b = 0; b < D / 64; ++b)
                    tma_store_3d(m128 + 1, src + b * 16384 + (a + i) * 128, b * 64, y + i, head);
        }
        r = seg_end;
    }
    bulk_commit();
    bulk_wait_read0();
}

template <int D, int CG>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_tc(const __grid_constant__ TcParams p) {
    using L = Layout<D, CG>;
    constexpr int NBOX = D / 64;
    constexpr int kKRows = kBN / CG;                        // key rows of this CTA's K part
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ = s_base + L::kQ;
    const uint32_t sKV = s_base + L::kKV;
    const uint32_t bars = s_base + L::kBars;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA pair: rank 0 issues every MMA for both CTAs; loads and P hand-offs
    // of both CTAs count on rank 0's barriers (`lead`).
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
    auto lead = [&](int i) -> uint32_t { return CG == 2 ? mapa_shared(bar(i), 0) : bar(i); };
    auto wait = [&](uint32_t b, uint32_t parity) -> bool {
        return CG == 2 ? mbar_wait_cluster(b, parity, kWaitNs) : mbar_wait(b, parity, kWaitNs);
    };

    if (threadIdx.x == 0) {
        mbar_init(bar(L::bQ), 1);
        mbar_init(bar(L::bQfree), 2);          // one arrive per softmax group
        // A slot is free once its MMAs completed (bEmpty) and, if it held a
        // chunk tile this CTA writes out, once both chunk-write warps have
        // copied it (bCopied).  bGo tells the chunk-write warps that such a
        // tile has landed: its phases advance only with copied loads, so a
        // parity wait on it always names the right load.
        for (int i = 0; i < L::kSlots; ++i) {
            mbar_init(bar(L::bFull + i), 1);
            mbar_init(bar(L::bEmpty + i), 1);
            mbar_init(bar(L::bCopied + i), p.commit_maps ? 1 : 2);   // TMA: one thread; else both warps
            mbar_init(bar(L::bGo + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(L::bS + i), 1);
            mbar_init(bar(L::bP + i), 4 * CG); // one arrive per softmax warp of the cluster
            mbar_init(bar(L::bPh + i), 4 * CG); // the same, once P of the tile's first 64 keys is stored
            mbar_init(bar(L::bO + i), 1);
            mbar_init(bar(L::bEpi + i), kBM);  // every softmax thread
        }
        mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_o);
        prefetch_tmap(CG == 2 ? &p.tm_k0h : &p.tm_k0);
        prefetch_tmap(&p.tm_v0);
        prefetch_tmap(CG == 2 ? &p.tm_k1h : &p.tm_k1);
        prefetch_tmap(&p.tm_v1);
    }
    if (warp == 1) {
        if (CG == 2) {
            tmem_alloc_pair(smem_u32(tmem_holder), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_holder), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();               // the peer's barriers exist before anything signals them
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // Registers: the producer / MMA warpgroup gives up what the softmax
    // warpgroups take: 4*32*(168-RTR_REGS_LOW) == 8*32*(RTR_REGS_HIGH-168).
    if (warp < 4) {
    set_max_regs_dec<RTR_REGS_LOW>();
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && !p.test_skip_loads) {
            Sched sc;
            Item it;
            int n = 0, k = 0;
            unsigned copy_pending = 0;     // slots whose last load the chunk-write warps copy out
            unsigned copy_phase = 0;       // per slot (bit), parity of its next bCopied phase
            bool ok = true;
            while (ok && sched_next<CG>(p, sc, it)) {
                int unit_row, head;
                unit_coords(p, it.unit, unit_row, head);
                const int q0 = unit_row * p.unit_rows;            // first row of the unit
                const int my_q0 = q0 + (int)rank * kPairRows;     // this CTA's rows
                if (k > 0 && !mbar_wait(bar(L::bQfree), (k - 1) & 1, kWaitNs)) {
                    raise_timeout(p, abort_flag);
                    break;
                }
                if (rank == 0) mbar_arrive_tx(bar(L::bQ), CG * 2 * L::kTileBytes);
                for (int i = 0; i < 2; ++i)
                    for (int b = 0; b < NBOX; ++b) {
                        if (CG == 2)
                            tma_load_3d_pair(sQ + i * L::kTileBytes + b * 16384, &p.tm_q, lead(L::bQ), b * 64, head,
                                             my_q0 + i * kBM);
                        else
                            tma_load_3d(sQ + i * L::kTileBytes + b * 16384, &p.tm_q, bar(L::bQ), b * 64, head,
                                        my_q0 + i * kBM);
                    }
                int s, tt;
                locate_tile(p, q0, it.t0, s, tt);
                int ntile = seg_tiles(p, s, q0);
                for (int t = it.t0; t < it.t1 && ok; ++t) {
                    while (tt >= ntile) {
                        ++s;
                        tt = 0;
                        ntile = seg_tiles(p, s, q0);
                    }
                    const KvSeg g = p.seg[s];
                    const int row = g.row0 + tt * kBN;
                    const bool copied = p.commit_k != nullptr && g.src == 1 && (tt >> 1) == unit_row;
                    for (int kv = 0; kv < 2; ++kv, ++n) {
                        const int slot = n % L::kSlots, use = n / L::kSlots;
                        if (*abort_flag) { ok = false; break; }
                        if (use > 0 && !mbar_wait(bar(L::bEmpty + slot), (use - 1) & 1, kWaitNs)) {
                            raise_timeout(p, abort_flag);
                            ok = false;
                            break;
                        }
                        if (copy_pending & (1u << slot)) {
                            if (!mbar_wait(bar(L::bCopied + slot), (copy_phase >> slot) & 1, kWaitNs)) {
                                raise_timeout(p, abort_flag);
                                ok = false;
                                break;
                            }
                            copy_phase ^= 1u << slot;
                        }
                        copy_pending = copied ? (copy_pending | (1u << slot)) : (copy_pending & ~(1u << slot));
                        const uint32_t dst = sKV + slot * L::kSlotBytes;
                        if (rank == 0) mbar_arrive_tx(bar(L::bFull + slot), CG * L::kSlotBytes);
                        if (CG == 1) {
                            const CUtensorMap *map =
                                g.src == 0 ? (kv ? &p.tm_v0 : &p.tm_k0) : (kv ? &p.tm_v1 : &p.tm_k1);
                            for (int b = 0; b < NBOX; ++b) {
                                if (g.src == 0)
                                    tma_load_3d(dst + b * 16384, map, bar(L::bFull + slot), b * 64, row, head);
                                else
                                    tma_load_3d(dst + b * 16384, map, bar(L::bFull + slot), b * 64, head, row);
                            }
                        } else if (kv == 0) {
                            // K: this CTA's half of the key rows, all of d
                            const CUtensorMap *map = g.src == 0 ? &p.tm_k0h : &p.tm_k1h;
                            const int r = row + (int)rank * kKRows;
                            for (int b = 0; b < NBOX; ++b) {
                                const uint32_t d_b = dst + b * (kKRows * 128);
                                if (g.src == 0)
                                    tma_load_3d_pair(d_b, map, lead(L::bFull + slot), b * 64, r, head);
                                else
                                    tma_load_3d_pair(d_b, map, lead(L::bFull + slot), b * 64, head, r);
                            }
                        } else {
                            // V: all key rows, this CTA's half of d (64 columns)
                            const CUtensorMap *map = g.src == 0 ? &p.tm_v0 : &p.tm_v1;
                            if (g.src == 0)
                                tma_load_3d_pair(dst, map, lead(L::bFull + slot), (int)rank * 64, row, head);
                            else
                                tma_load_3d_pair(dst, map, lead(L::bFull + slot), (int)rank * 64, head, row);
                        }
                    }
                    ++tt;
                }
                ++k;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM * CG, kBN, 0, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM * CG, D, 0, 1);
            // Descriptors depend only on the buffer: build them once, then
            // step along K by adding the byte offset >> 4 to the start-address
            // field (no carry: every address is below 256 KB).  In pair mode the
            // same offsets address the peer CTA's half of each operand.
            const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dq1 = smem_desc_sw128(sQ + L::kTileBytes, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sKV, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sKV, 16384, 1024);
            auto issue_s = [&](int i, int slot) {
                const uint64_t a0 = i ? dq1 : dq0;
                const uint64_t b0 = dk0 + (uint64_t)((slot * L::kSlotBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t a_off = ((kk / 4) * 16384 + (kk % 4) * 32) >> 4;
                    const uint32_t b_off = ((kk / 4) * (kKRows * 128) + (kk % 4) * 32) >> 4;
                    if (CG == 2)
                        mma_ss_pair(tmem + i * 128, a0 + a_off, b0 + b_off, idesc_s, kk > 0 ? 1u : 0u);
                    else
                        mma_ss(tmem + i * 128, a0 + a_off, b0 + b_off, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // PV over key steps [kk0, kk1) of 16 keys (all of them unless split)
            auto issue_pv = [&](int i, int slot, bool acc, int kk0 = 0, int kk1 = kBN / 16) {
                const uint64_t b0 = dv0 + (uint64_t)((slot * L::kSlotBytes) >> 4);
#pragma unroll
                for (int kk = kk0; kk < kk1; ++kk) {
                    if (CG == 2)
                        mma_ts_pair(tmem + 256 + i * D, tmem + i * 128 + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4),
                                    idesc_o, (acc || kk > 0) ? 1u : 0u);
                    else
                        mma_ts(tmem + 256 + i * D, tmem + i * 128 + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4),
                               idesc_o, (acc || kk > 0) ? 1u : 0u);
                }
            };
            auto commit = [&](int i) {
                if (CG == 2) tc_commit_pair(bar(i));
                else tc_commit(bar(i));
            };
            Sched sc;
            Item it;
            int n = 0, k = 0, jj = 0;   // ring loads consumed, items, tiles (S/P phases)
            bool ok = true;
            while (ok && sched_next<CG>(p, sc, it)) {
                const int T = it.t1 - it.t0;
                // Unit tiles from copy_lo on are the chunk's; those with chunk
                // tile (t - copy_lo) / 2 == the unit's pair index are copied out.
                int copy_lo = 1 << 30, copy_hi = 0, copy_pair = 0;
                if (p.commit_k != nullptr) {
                    int head_m;
                    unit_coords(p, it.unit, copy_pair, head_m);
                    const int q0m = copy_pair * p.unit_rows;
                    copy_lo = 0;                               // tiles of the runs before the chunk's
                    int s = 0;
                    for (; s < p.nseg && p.seg[s].src != 1; ++s) copy_lo += seg_tiles(p, s, q0m);
                    copy_hi = s < p.nseg ? copy_lo + seg_tiles(p, s, q0m) : copy_lo;
                }
                // [copy_lo, copy_hi) bounds the chunk's tiles: with an odd
                // tile count the tile after the chunk would otherwise match.
                auto go = [&](int t, int slot_) {
                    if (t >= copy_lo && t < copy_hi && ((t - copy_lo) >> 1) == copy_pair)
                        mbar_arrive(bar(L::bGo + slot_));
                };
                ok = wait(bar(L::bQ), k & 1) && !*abort_flag;
                if (!ok) break;
                int slot = n % L::kSlots;
                ok = wait(bar(L::bFull + slot), (n / L::kSlots) & 1);
                if (!ok) break;
                go(it.t0, slot);
                tc_fence_after();
                int kslot = slot;
                issue_s(0, kslot);
                commit(L::bS + 0);
                issue_s(1, kslot);
                commit(L::bS + 1);
                commit(L::bEmpty + slot);
                ++n;
                for (int j = 0; j < T; ++j, ++jj) {
                    const int vs = n % L::kSlots;
                    ok = wait(bar(L::bFull + vs), (n / L::kSlots) & 1);
                    if (!ok) break;
                    go(it.t0 + j, vs);
                    ++n;
                    const int vslot = vs;
                    int ks = -1;
                    if (RTR_PV_SPLIT) {
                        ok = wait(bar(L::bPh + 0), jj & 1) && !*abort_flag;
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(0, vslot, j > 0, 0, kBN / 32);
                    }
                    ok = wait(bar(L::bP + 0), jj & 1) && !*abort_flag;
                    if (!ok) break;
                    tc_fence_after();
                    if (RTR_PV_SPLIT)
                        issue_pv(0, vslot, true, kBN / 32, kBN / 16);
                    else
                        issue_pv(0, vslot, j > 0);
                    if (j == T - 1) commit(L::bO + 0);
                    if (j + 1 < T) {
                        ks = n % L::kSlots;
                        ok = wait(bar(L::bFull + ks), (n / L::kSlots) & 1);
                        if (!ok) break;
                        go(it.t0 + j + 1, ks);
                        tc_fence_after();
                        kslot = ks;
                        issue_s(0, kslot);
                        commit(L::bS + 0);
                    }
                    if (RTR_PV_SPLIT) {
                        ok = wait(bar(L::bPh + 1), jj & 1) && !*abort_flag;
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(1, vslot, j > 0, 0, kBN / 32);
                    }
                    ok = wait(bar(L::bP + 1), jj & 1) && !*abort_flag;
                    if (!ok) break;
                    tc_fence_after();
                    if (RTR_PV_SPLIT)
                        issue_pv(1, vslot, true, kBN / 32, kBN / 16);
                    else
                        issue_pv(1, vslot, j > 0);
                    commit(L::bEmpty + vs);
                    if (j == T - 1) commit(L::bO + 1);
                    if (j + 1 < T) {
                        issue_s(1, kslot);
                        commit(L::bS + 1);
                        commit(L::bEmpty + ks);
                        ++n;
                    }
                }
                ++k;
            }
            if (!ok) raise_timeout(p, abort_flag);
            // Drain: every MMA issued above has completed before TMEM is freed
            // (in pair mode the commit also releases the peer CTA).
            commit(L::bDrain);
            mbar_wait(bar(L::bDrain), 0, kWaitNs);
        } else if (lane == 0) {
            // pair mode, rank 1: wait until rank 0's MMAs into this CTA's TMEM are done
            mbar_wait(bar(L::bDrain), 0, kWaitNs);
        }
        __syncwarp();
    } else if (warp >= 2 && p.commit_k != nullptr && (p.commit_maps == nullptr || (warp == 2 && lane == 0))) {
        // ------------------------------------------------------------ chunk write
        // Walks the producer's load sequence and waits (on bGo) only for the
        // loads it copies.  Chunk key tile tt belongs to the unit of query tiles 2u,
        // 2u+1 with u = tt / 2 (that unit always loads it), so every chunk
        // tile is written by exactly one CTA.  The producer refills such a
        // slot only after both warps arrived on its bCopied barrier.
        // With store maps, lane 0 of warp 2 alone issues TMA stores;
        // otherwise both warps copy half of each tile's rows.
        const bool tma = p.commit_maps != nullptr;
        const int part = warp - 2;
        Sched sc;
        Item it;
        int n = 0;
        unsigned go_phase = 0;         // per slot (bit), parity of its next bGo phase
        bool ok = true;
        while (ok && sched_next<CG>(p, sc, it)) {
            int unit_row, head;
            unit_coords(p, it.unit, unit_row, head);
            const int q0 = unit_row * p.unit_rows;
            int s, tt;
            locate_tile(p, q0, it.t0, s, tt);
            int ntile = seg_tiles(p, s, q0);
            for (int t = it.t0; t < it.t1 && ok; ++t, ++tt) {
                while (tt >= ntile) {
                    ++s;
                    tt = 0;
                    ntile = seg_tiles(p, s, q0);
                }
                const bool mine = p.seg[s].src == 1 && (tt >> 1) == unit_row;
                if (!mine) {
                    n += 2;
                    continue;
                }
                for (int kv = 0; kv < 2; ++kv, ++n) {
                    const int slot = n % L::kSlots;
                    bool w = !*abort_flag && mbar_wait(bar(L::bGo + slot), (go_phase >> slot) & 1, kWaitNs);
                    if (!tma) w = __all_sync(0xffffffffu, w);
                    if (!w) { ok = false; break; }
                    go_phase ^= 1u << slot;
                    if (tma) {
                        commit_tile_tma<D>(p, sKV + slot * L::kSlotBytes, kv, head, tt);
                        mbar_arrive(bar(L::bCopied + slot));
                    } else {
                        commit_tile_rows<D>(p, sKV + slot * L::kSlotBytes, kv ? p.commit_v : p.commit_k, head, tt,
                                            part, lane);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(L::bCopied + slot));
                    }
                }
            }
        }
        if (!ok) raise_timeout(p, abort_flag);
    }
    } else {
        set_max_regs_inc<RTR_REGS_HIGH>();
        // ------------------------------------------------------------ softmax
        const int i = (warp - 4) >> 2;                  // which query tile of the pair
        const int sub = warp & 3;                       // TMEM lane quarter
        const int row_local = sub * 32 + lane;
        const uint32_t lane_bits = (uint32_t)(sub * 32) << 16;
        const uint32_t tS = tmem + lane_bits + i * 128;
        const uint32_t tO = tmem + lane_bits + 256 + i * D;
        const uint32_t sOut = sQ + i * L::kTileBytes;   // Q_i is dead once O_i is final
        const float sl2 = p.scale_log2;
        Sched sc;
        Item it;
        int k = 0, jj = 0;
        bool ok = true;
        while (ok && sched_next<CG>(p, sc, it)) {
            int unit_row, head;
            unit_coords(p, it.unit, unit_row, head);
            const int q0 = unit_row * p.unit_rows;              // first row of the unit
            const int my_q0 = q0 + (int)rank * kPairRows;       // this CTA's rows
            const int q_row = my_q0 + i * kBM + row_local;
            const int row_vis_end = (q_row / p.kpf + 1) * p.kpf;
            float m_run = -INFINITY, l_run = 0.f;
            int s, tt;
            locate_tile(p, q0, it.t0, s, tt);
            int ntile = seg_tiles(p, s, q0);
            for (int t = it.t0; t < it.t1; ++t, ++jj, ++tt) {
                while (tt >= ntile) {
                    ++s;
                    tt = 0;
                    ntile = seg_tiles(p, s, q0);
                }
                const KvSeg g = p.seg[s];
                const int row_len = g.causal ? min(g.len, row_vis_end) : g.len;
                const int lim = row_len - tt * kBN;     // visible columns of this row
                bool w = !*abort_flag && mbar_wait(bar(L::bS + i), jj & 1, kWaitNs);
                w = __all_sync(0xffffffffu, w);
                if (!w) { ok = false; break; }
                tc_fence_after();
                // Warp-uniform: the code below holds tcgen05 .sync.aligned
                // instructions, which every lane of the warp must execute together.
                const bool masked = __any_sync(0xffffffffu, lim < kBN);
#if RTR_SOFTMAX_1LD
                // The row's 128 scores in registers: one TMEM read, the max,
                // then P over them in four 32-column chunks.
                uint32_t sr[128];
                tmem_ld128(tS, sr);
                tmem_wait_ld();
                if (masked) {
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        if (e >= lim) sr[e] = __float_as_uint(-INFINITY);
                }
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int e = 0; e < 128; e += 8) {
                    mx0 = max3f(mx0, __uint_as_float(sr[e + 0]), __uint_as_float(sr[e + 1]));
                    mx1 = max3f(mx1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
                    mx2 = max3f(mx2, __uint_as_float(sr[e + 4]), __uint_as_float(sr[e + 5]));
                    mx3 = max3f(mx3, __uint_as_float(sr[e + 6]), __uint_as_float(sr[e + 7]));
                }
#else
                // Pass 1: row max, 64 columns per TMEM round trip (the row is read
                // again in pass 2 instead of being held in registers).
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t ra[32], rb[32];
                    tmem_ld32(tS + 64 * h, ra);
                    tmem_ld32(tS + 64 * h + 32, rb);
                    tmem_wait_ld();
                    if (masked) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (64 * h + e >= lim) ra[e] = __float_as_uint(-INFINITY);
                            if (64 * h + 32 + e >= lim) rb[e] = __float_as_uint(-INFINITY);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        mx0 = max3f(mx0, __uint_as_float(ra[e + 0]), __uint_as_float(ra[e + 1]));
                        mx1 = max3f(mx1, __uint_as_float(ra[e + 2]), __uint_as_float(ra[e + 3]));
                        mx2 = max3f(mx2, __uint_as_float(ra[e + 4]), __uint_as_float(ra[e + 5]));
                        mx3 = max3f(mx3, __uint_as_float(ra[e + 6]), __uint_as_float(ra[e + 7]));
                        mx0 = max3f(mx0, __uint_as_float(rb[e + 0]), __uint_as_float(rb[e + 1]));
                        mx1 = max3f(mx1, __uint_as_float(rb[e + 2]), __uint_as_float(rb[e + 3]));
                        mx2 = max3f(mx2, __uint_as_float(rb[e + 4]), __uint_as_float(rb[e + 5]));
                        mx3 = max3f(mx3, __uint_as_float(rb[e + 6]), __uint_as_float(rb[e + 7]));
                    }
                }
#endif
                const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
                const float m_new = fmaxf(m_run, mx * sl2);
                const bool upd = m_new > m_run + 8.0f;
                float factor = 1.f;
                if (upd) {
                    factor = fast_exp2(m_run - m_new);
                    m_run = m_new;
                    l_run *= factor;
                }
                if (t > it.t0 && __any_sync(0xffffffffu, upd)) {
#if RTR_SOFTMAX_1LD
                    // 16 columns at a time: the row's scores are still live
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        uint32_t o[16];
                        tmem_ld16(tO + 16 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                        tmem_st16(tO + 16 * c, o);
                    }
#else
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                        tmem_st32(tO + 32 * c, o);
                    }
#endif
                }
                const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f)};
                // Pass 2: P for 32 columns per step, the next 32 loading while
                // these are computed; P (bf16 pairs) goes over the row's first
                // 64 columns, behind the scores already read.  The polynomial
                // exp2 runs only on tiles without masked entries (every input
                // finite); ex2 maps -inf to exactly 0.
#if RTR_SOFTMAX_1LD
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    if (masked) softmax_chunk_regs<false>(sr + 32 * q4, sl2, neg_m, tS + 16 * q4, acc);
                    else softmax_chunk_regs<true>(sr + 32 * q4, sl2, neg_m, tS + 16 * q4, acc);
                    if (RTR_PV_SPLIT && q4 == 1) {
                        // P of the first 64 keys is in TMEM: their PV may start
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (CG == 2) mbar_arrive_cluster(lead(L::bPh + i));
                            else mbar_arrive(bar(L::bPh + i));
                        }
                    }
                }
#else
                {
                    uint32_t buf[2][32];
                    tmem_ld32(tS, buf[0]);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        if (q4 < 3) tmem_ld32(tS + 32 * (q4 + 1), buf[(q4 + 1) & 1]);
                        if (masked) {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (32 * q4 + e >= lim) buf[q4 & 1][e] = __float_as_uint(-INFINITY);
                            softmax_chunk<false>(buf[q4 & 1], sl2, neg_m, tS + 16 * q4, acc);
                        } else {
                            softmax_chunk<true>(buf[q4 & 1], sl2, neg_m, tS + 16 * q4, acc);
                        }
                        if (q4 < 3) tmem_wait_ld();
                        if (RTR_PV_SPLIT && q4 == 1) {
                            // P of the first 64 keys is in TMEM: their PV may start
                            tmem_wait_st();
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) {
                                if (CG == 2) mbar_arrive_cluster(lead(L::bPh + i));
                                else mbar_arrive(bar(L::bPh + i));
                            }
                        }
                    }
                }
#endif
                const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
                const float2 a4 = fadd2(a01, a23);
                l_run += a4.x + a4.y;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (CG == 2) mbar_arrive_cluster(lead(L::bP + i));
                    else mbar_arrive(bar(L::bP + i));
                }
            }
            if (!ok) break;
            // -------------------------------------------------------- epilogue
            bool w = !*abort_flag && mbar_wait(bar(L::bO + i), k & 1, kWaitNs);
            w = __all_sync(0xffffffffu, w);
            if (!w) { ok = false; break; }
            tc_fence_after();
            const int prow = i * kBM + row_local;       // row within the pair
            if (it.slot < 0 && p.out_f32 != nullptr) {
                // fp32 output: the normalised row straight to global memory
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                if (p.lse != nullptr && q_row < p.nq)
                    p.lse[(size_t)head * p.nq + q_row] =
                        l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
                float4 *dst = reinterpret_cast<float4 *>(p.out_f32 + ((size_t)q_row * p.heads + head) * D);
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
                    if (q_row < p.nq) {
#pragma unroll
                        for (int t4 = 0; t4 < 8; ++t4)
                            dst[8 * c + t4] = make_float4(
                                __uint_as_float(o[4 * t4 + 0]) * inv, __uint_as_float(o[4 * t4 + 1]) * inv,
                                __uint_as_float(o[4 * t4 + 2]) * inv, __uint_as_float(o[4 * t4 + 3]) * inv);
                    }
                }
            } else if (it.slot < 0) {
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                if (p.lse != nullptr && q_row < p.nq)
                    p.lse[(size_t)head * p.nq + q_row] =
                        l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int t4 = 0; t4 < 4; ++t4) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(o[8 * t4 + 0]) * inv, __uint_as_float(o[8 * t4 + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(o[8 * t4 + 2]) * inv, __uint_as_float(o[8 * t4 + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(o[8 * t4 + 4]) * inv, __uint_as_float(o[8 * t4 + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(o[8 * t4 + 6]) * inv, __uint_as_float(o[8 * t4 + 7]) * inv);
                        const int col = 32 * c + 8 * t4;
                        const int box = col / 64, cc = (col % 64) / 8;
                        const uint32_t addr = sOut + box * 16384 + row_local * 128 + ((cc ^ (row_local & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                                     "r"(v.z), "r"(v.w)
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
            } else {
                // Partial: unnormalised O, running max and row sum, laid out so
                // that consecutive rows are consecutive float4s.
                const size_t base = ((size_t)blockIdx.x * 2 + it.slot);
                float4 *po = p.part_o + base * (D / 4) * kPairRows;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int t4 = 0; t4 < 8; ++t4)
                        po[(size_t)(8 * c + t4) * kPairRows + prow] =
                            make_float4(__uint_as_float(o[4 * t4 + 0]), __uint_as_float(o[4 * t4 + 1]),
                                        __uint_as_float(o[4 * t4 + 2]), __uint_as_float(o[4 * t4 + 3]));
                }
                p.part_ml[base * kPairRows + prow] = make_float2(m_run, l_run);
            }
            tc_fence_before();
            mbar_arrive(bar(L::bEpi + i));
            if (row_local == 0) {
                const bool all = mbar_wait(bar(L::bEpi + i), k & 1, kWaitNs);
                if (!all) raise_timeout(p, abort_flag);
                if (all && it.slot < 0 && p.out_f32 == nullptr && my_q0 + i * kBM < p.nq) {
                    for (int b = 0; b < NBOX; ++b)
                        tma_store_3d(&p.tm_o, sOut + b * 16384, b * 64, head, my_q0 + i * kBM);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(bar(L::bQfree));
            }
            ++k;
        }
        if (!ok) raise_timeout(p, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();               // neither CTA leaves while the pair's MMAs may touch it
    if (warp == 1) {
        tc_fence_after();
        if (CG == 2) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

// Merge the partial results of units split across clusters.  Grid: (units of
// the shared remainder, CG * 4); each block covers 64 query rows of one CTA's
// share of a unit, each thread one row and a quarter of the head dimension.
template <int D, int CG>
__global__ void __launch_bounds__(256) attn_combine(const __grid_constant__ TcParams p) {
    const int ru = p.full_rounds * p.grid + blockIdx.x;
    if (ru >= p.n_units) return;
    const long long U = p.rem_U[blockIdx.x];
    int unit_row, head;
    unit_coords(p, ru, unit_row, head);
    const int T = pair_tiles(p, unit_row);
    // cluster whose range holds tile x: rem_lo[c] <= x < rem_lo[c+1]
    auto owner = [&](long long x) {
        int lo = 0, hi = p.grid - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (p.rem_lo[mid] <= x) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    const int c0 = owner(U), c1 = owner(U + T - 1);
    if (c0 == c1) return;                           // whole unit: written by its cluster
    const int r = blockIdx.y / 4;                   // CTA of the cluster
    const int row = (blockIdx.y % 4) * 64 + (threadIdx.x >> 2);   // row within that CTA's share
    const int quarter = threadIdx.x & 3;            // D/4 columns each
    const int q = unit_row * p.unit_rows + r * kPairRows + row;
    if (q >= p.nq) return;
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c) {
        if (p.rem_lo[c] == p.rem_lo[c + 1]) continue;
        const int slot = (c == c0 && U != p.rem_lo[c0]) ? 1 : 0;
        M = fmaxf(M, p.part_ml[((size_t)(c * CG + r) * 2 + slot) * kPairRows + row].x);
    }
    constexpr int NV = D / 16;                       // float4 per thread
    float l = 0.f;
    float4 acc[NV];
#pragma unroll
    for (int e = 0; e < NV; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = c0; c <= c1; ++c) {
        if (p.rem_lo[c] == p.rem_lo[c + 1]) continue;
        const int slot = (c == c0 && U != p.rem_lo[c0]) ? 1 : 0;
        const size_t base = (size_t)(c * CG + r) * 2 + slot;
        const float2 ml = p.part_ml[base * kPairRows + row];
        const float w = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
        l += w * ml.y;
        const float4 *po = p.part_o + base * (D / 4) * kPairRows;
#pragma unroll
        for (int e = 0; e < NV; ++e) {
            const float4 v = po[(size_t)(quarter * NV + e) * kPairRows + row];
            acc[e].x += w * v.x;
            acc[e].y += w * v.y;
            acc[e].z += w * v.z;
            acc[e].w += w * v.w;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (p.lse != nullptr && quarter == 0)
        p.lse[(size_t)head * p.nq + q] = l > 0.f ? (M + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (p.out_f32 != nullptr) {
        float4 *df = reinterpret_cast<float4 *>(p.out_f32 + ((size_t)q * p.heads + head) * D + quarter * (D / 4));
#pragma unroll
        for (int e = 0; e < NV; ++e)
            df[e] = make_float4(acc[e].x * inv, acc[e].y * inv, acc[e].z * inv, acc[e].w * inv);
        return;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)q * p.heads + head) * D + quarter * (D / 4));
#pragma unroll
    for (int e = 0; e < NV / 2; ++e) {
        uint4 v;
        v.x = pack_bf16x2(acc[2 * e].x * inv, acc[2 * e].y * inv);
        v.y = pack_bf16x2(acc[2 * e].z * inv, acc[2 * e].w * inv);
        v.z = pack_bf16x2(acc[2 * e + 1].x * inv, acc[2 * e + 1].y * inv);
        v.w = pack_bf16x2(acc[2 * e + 1].z * inv, acc[2 * e + 1].w * inv);
        dst[e] = v;
    }
}

template <int D, int CG>
cudaError_t launch_tc(const TcParams &tp, bool has_split, cudaStream_t s) {
    using L = Layout<D, CG>;
    static std::atomic<unsigned> configured_mask{0};   // per device bit (up to 32 devices)
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned bit = 1u << (dev & 31);
    if (!(configured_mask.load(std::memory_order_acquire) & bit)) {
        // two threads may both set the attribute; the call is idempotent
        cudaError_t e =
            cudaFuncSetAttribute(attn_fwd_tc<D, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return e;
        configured_mask.fetch_or(bit, std::memory_order_release);
    }
    cudaError_t e;
    if (CG == 2) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(tp.grid * 2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = L::kAlloc;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, attn_fwd_tc<D, CG>, tp);
    } else {
        attn_fwd_tc<D, CG><<<tp.grid, kThreads, L::kAlloc, s>>>(tp);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    count_launch();
    const int rem_units = tp.n_units - tp.full_rounds * tp.grid;
    if (rem_units > 0 && has_split) {
        attn_combine<D, CG><<<dim3(rem_units, CG * 4), 256, 0, s>>>(tp);
        e = cudaGetLastError();
        if (e == cudaSuccess) count_launch();
    }
    return e;
}

// Host copy of the device's tile count per unit (rows [idx*unit_rows, ...)).
int host_pair_tiles(const AttnProblem &p, int idx, int unit_rows) {
    int t = 0;
    const int q0 = idx * unit_rows;
    for (int s = 0; s < p.nseg; ++s) {
        int len = p.seg[s].len;
        if (p.seg[s].causal) {
            const int q_last = std::min(q0 + unit_rows - 1, p.nq - 1);
            const int lim = (q_last / p.kpf + 1) * p.kpf;
            len = std::min(len, lim);
        }
        t += (len + kBN - 1) / kBN;
    }
    return t;
}

}  // namespace

// Device address of g_device_status on `device` (which must be current),
// looked up once per device under a lock: two host threads making their
// first call at the same time both get the same address.
unsigned *device_status_ptr(int device) {
    static std::mutex mu;
    static unsigned *ptrs[64] = {};
    if (device < 0 || device >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[device]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        ptrs[device] = static_cast<unsigned *>(p);
    }
    return ptrs[device];
}

// Scheduling of the persistent kernel (mirrors sched_next on the device):
// full rounds of one unit per CTA, then the remaining units' key tiles cut
// into per-CTA ranges sized so that every CTA's total (its full-round units
// plus its range) is as equal as possible.
void plan_attn_bf16(const AttnProblem &p, int sms, int cg, AttnPlan &plan) {
    plan.cg = (cg == 2 && p.head_dim == 128) ? 2 : 1;
    plan.unit_rows = kPairRows * plan.cg;
    plan.n_pairs = (p.nq + plan.unit_rows - 1) / plan.unit_rows;
    plan.n_units = plan.n_pairs * p.heads;
    const int G = std::max(1, std::min(sms / plan.cg, kMaxGrid));   // clusters
    plan.full_rounds = plan.n_units / G;
    std::vector<int> pt(plan.n_pairs);
    int tmin = 1 << 30, tmax = 0;
    for (int pr = 0; pr < plan.n_pairs; ++pr) {
        pt[pr] = host_pair_tiles(p, pr, plan.unit_rows);
        tmin = std::min(tmin, pt[pr]);
        tmax = std::max(tmax, pt[pr]);
    }
    plan.head_major = (double)tmax <= RTR_UNIT_ORDER_RATIO * (double)tmin ? 1 : 0;
    auto unit_T = [&](int u) {
        const int pair = plan.head_major ? plan.n_pairs - 1 - u % plan.n_pairs : plan.n_pairs - 1 - u / p.heads;
        return pt[pair];
    };
    long long rem_total = 0;
    for (int u = plan.full_rounds * G; u < plan.n_units; ++u) rem_total += unit_T(u);
    std::vector<long long> load(G, 0);
    long long total = rem_total;
    for (int c = 0; c < G; ++c)
        for (int r = 0; r < plan.full_rounds; ++r) {
            load[c] += unit_T(full_round_unit(G, c, r));
            total += unit_T(full_round_unit(G, c, r));
        }
    long long budget = (total + G - 1) / G;
    // A split part costs a Q load and an epilogue: with no full rounds, give
    // each CTA at least 8 key tiles.
    if (plan.full_rounds == 0) budget = std::max<long long>(budget, 8);
    // The alternative: the remaining units whole, unit i to CTA i (when they
    // are no more than the CTAs).  Splitting evens the CTAs' totals out, but
    // every split part pays a work item's fixed cost (its Q load, the first
    // S before any softmax, its epilogue: measured at roughly 8 key-tile
    // steps) and the partial results need the combine kernel (about 7 more).
    // For short units (cross attention over 4 key tiles, single-frame chunks)
    // whole units finish first.
    const int R = plan.n_units - plan.full_rounds * G;
    bool whole = false;
    if (R > 0 && R <= G) {
        long long make_whole = 0;
        for (int c = 0; c < G; ++c)
            make_whole = std::max(make_whole, load[c] + (c < R ? unit_T(plan.full_rounds * G + c) : 0));
        whole = make_whole <= budget + kSplitPenaltyTiles;
    }
    plan.rem_lo.assign(G + 1, 0);
    if (whole) {
        for (int c = 0; c < G; ++c)
            plan.rem_lo[c + 1] = plan.rem_lo[c] + (c < R ? unit_T(plan.full_rounds * G + c) : 0);
    } else {
        for (int c = 0; c < G; ++c) {
            const long long share = std::max<long long>(0, budget - load[c]);
            plan.rem_lo[c + 1] = (int)std::min(rem_total, plan.rem_lo[c] + share);
        }
    }
    plan.grid = G;
    if (plan.full_rounds == 0) {
        int used = 1;
        while (used < G && plan.rem_lo[used] < rem_total) ++used;
        plan.grid = used;
        plan.rem_lo.resize(used + 1);
    }
    plan.rem_lo.back() = (int)rem_total;
    // Tile offsets of the remainder units; any unit split across CTAs?
    plan.has_split = false;
    plan.rem_U.clear();
    long long U = 0;
    int c = 0;
    for (int u = plan.full_rounds * G; u < plan.n_units; ++u) {
        const int T = unit_T(u);
        plan.rem_U.push_back((int)U);
        while (c + 1 < plan.grid && plan.rem_lo[c + 1] <= U) ++c;
        if (U + T > plan.rem_lo[c + 1]) plan.has_split = true;
        U += T;
    }
    plan.scratch_bytes =
        (size_t)plan.cg * plan.grid * 2 * ((size_t)kPairRows * p.head_dim * 4 + (size_t)kPairRows * 8);
}

namespace {
std::atomic<int> g_inject_timeouts[64] = {};   // per device: launches left that skip their loads
}

void inject_wait_timeouts(int device, int launches) {
    if (device >= 0 && device < 64) g_inject_timeouts[device].store(launches > 0 ? launches : 0);
}

cudaError_t launch_attn_bf16(const AttnProblem &p, const AttnPlan &plan, const CUtensorMap *tm_k0,
                             const CUtensorMap *tm_k0h, const CUtensorMap *tm_v0, unsigned *status, void *scratch,
                             cudaStream_t s) {
    TcParams tp;
    memset(&tp, 0, sizeof(tp));
    int dev = 0;
    int left = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 &&
        (left = g_inject_timeouts[dev].load()) > 0 &&
        g_inject_timeouts[dev].compare_exchange_strong(left, left - 1)) {
        tp.test_skip_loads = 1;
    }
    const uint64_t D = (uint64_t)p.head_dim;
    if (!make_tmap_bf16(&tp.tm_q, p.q, D, p.heads, p.nq, 1, kBM)) return cudaErrorInvalidValue;
    // with an fp32 output the bf16 output map is never used: any valid map
    if (!make_tmap_bf16(&tp.tm_o, p.o_f32 ? p.q : p.o, D, p.heads, p.nq, 1, kBM)) return cudaErrorInvalidValue;
    bool have0 = false, have1 = false;
    for (int i = 0; i < p.nseg; ++i) (p.seg[i].src == 0 ? have0 : have1) = true;
    if (have1) {
        if (!make_tmap_bf16(&tp.tm_k1, p.k1, D, p.heads, p.rows1, 1, kBN)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16(&tp.tm_v1, p.v1, D, p.heads, p.rows1, 1, kBN)) return cudaErrorInvalidValue;
        if (plan.cg == 2 && !make_tmap_bf16(&tp.tm_k1h, p.k1, D, p.heads, p.rows1, 1, kBN / 2))
            return cudaErrorInvalidValue;
    } else {
        tp.tm_k1 = tp.tm_q;   // never read; any valid map
        tp.tm_v1 = tp.tm_q;
    }
    if (plan.cg != 2 || !have1) tp.tm_k1h = tp.tm_k1;
    if (have0) {
        tp.tm_k0 = *tm_k0;
        tp.tm_v0 = *tm_v0;
        if (plan.cg == 2 && !tm_k0h) return cudaErrorInvalidValue;
        tp.tm_k0h = tm_k0h ? *tm_k0h : *tm_k0;
    } else {
        tp.tm_k0 = tp.tm_q;
        tp.tm_v0 = tp.tm_q;
        tp.tm_k0h = tp.tm_q;
    }
    tp.nq = p.nq;
    tp.heads = p.heads;
    tp.kpf = p.kpf;
    tp.nseg = p.nseg;
    tp.unit_rows = plan.unit_rows;
    for (int i = 0; i < p.nseg; ++i) tp.seg[i] = p.seg[i];
    tp.scale_log2 = p.scale * 1.4426950408889634f;
    tp.status = status;
    tp.n_pairs = plan.n_pairs;
    tp.n_units = plan.n_units;
    tp.grid = plan.grid;
    tp.full_rounds = plan.full_rounds;
    tp.head_major = plan.head_major;
    if ((int)plan.rem_lo.size() != plan.grid + 1 || plan.grid > kMaxGrid) return cudaErrorInvalidValue;
    for (int c = 0; c <= plan.grid; ++c) tp.rem_lo[c] = plan.rem_lo[c];
    if (plan.rem_U.size() > (size_t)kMaxGrid) return cudaErrorInvalidValue;
    for (size_t i = 0; i < plan.rem_U.size(); ++i) tp.rem_U[i] = plan.rem_U[i];
    const size_t part_o_bytes = (size_t)plan.cg * plan.grid * 2 * kPairRows * p.head_dim * 4;
    tp.part_o = static_cast<float4 *>(scratch);
    tp.part_ml = reinterpret_cast<float2 *>(static_cast<char *>(scratch) + part_o_bytes);
    tp.out = static_cast<__nv_bfloat16 *>(p.o);
    tp.out_f32 = p.o_f32;
    if (p.o_f32 && (plan.cg != 1 || p.commit_k)) return cudaErrorInvalidValue;
    tp.lse = p.lse;
    if (p.commit_k) {
        // the chunk write is implemented for one CTA per MMA and needs the
        // chunk as the token-major run
        if (plan.cg != 1 || !p.commit_v || p.commit_slots < 1 || p.commit_first_slot < 0 ||
            p.commit_first_slot >= p.commit_slots || !have1)
            return cudaErrorInvalidValue;
        tp.commit_k = static_cast<__nv_bfloat16 *>(p.commit_k);
        tp.commit_v = static_cast<__nv_bfloat16 *>(p.commit_v);
        tp.commit_rows_per_head = p.rows0;
        tp.commit_first_slot = p.commit_first_slot;
        tp.commit_slots = p.commit_slots;
        tp.commit_row0 = p.commit_row0;
        tp.commit_maps = p.commit_maps;
    }
    if (p.head_dim == 128)
        return plan.cg == 2 ? launch_tc<128, 2>(tp, plan.has_split, s) : launch_tc<128, 1>(tp, plan.has_split, s);
    if (p.head_dim == 64) return launch_tc<64, 1>(tp, plan.has_split, s);
    return cudaErrorInvalidValue;
}

}  // namespace rtr
