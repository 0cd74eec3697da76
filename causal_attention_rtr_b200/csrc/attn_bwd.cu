// attn_bwd.cu -- backward pass of the block-causal attention on the
// 5th-generation tensor cores (sm_100a).
//
// The gradient of O = softmax(S) V, S = scale Q K^T + M, with the frame-causal
// mask M of RTR-DiT (papernotes.org note "DiT as Real-Time Rerenderer",
// Method > Key Designs 2; training by Self Forcing / DMD runs through it,
// Key Designs 3).  With P = softmax(S), the row log-sum-exp L saved by the
// forward (P_ij = exp(S_ij - L_i)) and Delta_i = sum_e dO_ie O_ie:
//
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   bwd_prep    Delta_i and L_i * log2(e) per (head, row), in [heads][n_pad]
//               fp32 scratch padded to whole 128-row tiles (padding: Delta 0,
//               L +inf, so padded query rows carry exactly zero probability).
//   bwd_dkdv    key-stationary: one CTA per (head, 128-key tile); streams the
//               query tiles that see it (frame-causal: query frames >= the
//               key tile's first frame).  Per query tile: S^T = K Q^T and
//               dP^T = V dO^T into TMEM (N = 128: the 64-wide forms of an
//               earlier half-tile version ran at a third of the tensor
//               core's rate); the softmax warps read the S^T row into
//               registers at once, which frees its columns for the next
//               tile's S^T, then write P^T and dS^T (bf16) over the dP^T
//               columns they have read; dV += P^T dO and dK += dS^T Q with
//               the "A in tensor memory" form, the first 64 queries' part
//               while the softmax does the other 64.
//   bwd_dq      query-stationary: one CTA per (head, 128-query tile); streams
//               the key tiles it sees (K through 3 shared-memory slots, V
//               through 2).  S = Q K^T into one of two TMEM buffers and
//               dP = dO V^T into one; the softmax reads the dP row into
//               registers at once, which frees dP's columns for the next
//               tile's dP, and writes dS (bf16) over S's columns; dQ += dS K,
//               the first 64 keys' part while the softmax does the rest.
// Splitting dQ from dK/dV recomputes S and dP once more (7 tile MMAs per
// (query tile, key tile) instead of 5) but needs no atomic accumulation of
// dQ across CTAs: every output tile is written once, in bf16, by TMA.
//
// One CTA, 256 threads: warp 0 TMA producer, warp 1 tcgen05 issuer (one
// thread), warps 4-7 softmax / epilogue (one thread per TMEM lane = row of
// the stationary tile).  Every wait is bounded (1 s) and a timeout latches
// RTR_E_TIMEOUT in the device status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace rtr {
namespace {

constexpr int kBT = 128;                  // rows of every tile
constexpr int kHalf = 64;                 // query columns after which bwd_dkdv starts dV / dK
constexpr int kDkdvThreads = 384;           // bwd_dkdv: producer, MMA, 2 idle, 8 softmax warps
constexpr int kDqThreads = 256;             // bwd_dq: producer, MMA, 2 idle, 4 softmax warps
constexpr uint64_t kBwdWaitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;   // token-major [n][H][D], box (64, 1, 128)
    CUtensorMap tm_dq, tm_dk, tm_dv;
    const float *delta;                    // [H][n_pad]
    const float *lse2;                     // [H][n_pad]: L * log2(e), +inf padding
    int n, n_pad, heads, kpf;
    float scale, scale_log2;
    unsigned *status;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Shared memory of bwd_dkdv: the stationary K and V tiles, then two stages
// of one streamed query tile each (Q and dO, 128 rows, plus 128 floats each
// of L*log2e and Delta), then the barriers.
template <int D>
struct DkdvLayout {
    static constexpr int kTile = kBT * D * 2;             // K, V, Q or dO
    static constexpr int kA = 0;                          // K, V
    static constexpr int kStage = 2 * kTile + 1024;       // Q, dO, L2[128], Delta[128]
    static constexpr int kB = 2 * kTile;                  // stage s at kB + s * kStage
    static constexpr int kBars = kB + 2 * kStage;
    static constexpr int bA = 0, bFull = 1, bEmpty = 3, bS = 5, bSread = 6, bPh = 7, bP = 8, bO = 9, bEpi = 10,
                         kNumBars = 11;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(DkdvLayout<128>::kAlloc <= 232448, "bwd_dkdv shared memory");

// Shared memory of bwd_dq: the stationary Q and dO tiles, then separate
// rings for K (3 slots) and V (2 slots).  K(t) is read by S(t) and by
// dQ(t), the last MMA of step t, so its slot frees late; a third K slot
// lets the load of K(t+3) start a full step before S(t+3) wants it.  V(t)
// is read by dP(t) alone and frees a step earlier, so two slots suffice.
template <int D>
struct DqLayout {
    static constexpr int kTile = kBT * D * 2;
    static constexpr int kKSlots = 3, kVSlots = 2;
    static constexpr int kA = 0;                          // Q, dO
    static constexpr int kK = 2 * kTile;                  // K slot s at kK + s * kTile
    static constexpr int kV = kK + kKSlots * kTile;       // V slot s at kV + s * kTile
    static constexpr int kBars = kV + kVSlots * kTile;
    static constexpr int bA = 0, bKFull = 1, bKEmpty = bKFull + kKSlots, bVFull = bKEmpty + kKSlots,
                         bVEmpty = bVFull + kVSlots, bS = bVEmpty + kVSlots, bDPread = bS + 1, bPh = bDPread + 1,
                         bP = bPh + 1, bO = bP + 1, bEpi = bO + 1, kNumBars = bEpi + 1;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(DqLayout<128>::kAlloc <= 232448, "bwd_dq shared memory");

__device__ __forceinline__ void bwd_timeout(const BwdParams &p, volatile int *abort_flag) {
    *abort_flag = 1;
    atomicExch(p.status, (unsigned)RTR_E_TIMEOUT);
}

// Load one 128-row tile of a token-major [n][H][D] tensor (D/64 boxes).
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap *map, uint32_t bar, int head, int row0) {
#pragma unroll
    for (int b = 0; b < D / 64; ++b) tma_load_3d(dst + b * 16384, map, bar, b * 64, head, row0);
}

// SS MMA chain over d: C[128 x N] = A[128 x D] B[N x D]^T, both K-major
// tiles in the TMA layout (B may start at a row offset inside its tile).
template <int D>
__device__ __forceinline__ void mma_tile_ss(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * 16384 + (kk % 4) * 32) >> 4;
        mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
    }
}



// Epilogue: 128 x D fp32 accumulator rows (this thread's TMEM lane) times
// `mul`, to bf16 in the swizzled TMA layout at `dst`.
template <int D>
__device__ __forceinline__ void acc_to_smem(uint32_t t_acc, float mul, uint32_t dst, int row) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_acc + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int t4 = 0; t4 < 4; ++t4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * t4 + 0]) * mul, __uint_as_float(o[8 * t4 + 1]) * mul);
            v.y = pack_bf16x2(__uint_as_float(o[8 * t4 + 2]) * mul, __uint_as_float(o[8 * t4 + 3]) * mul);
            v.z = pack_bf16x2(__uint_as_float(o[8 * t4 + 4]) * mul, __uint_as_float(o[8 * t4 + 5]) * mul);
            v.w = pack_bf16x2(__uint_as_float(o[8 * t4 + 6]) * mul, __uint_as_float(o[8 * t4 + 7]) * mul);
            const int col = 32 * c + 8 * t4;
            const int box = col / 64, cc = (col % 64) / 8;
            const uint32_t addr = dst + box * 16384 + row * 128 + ((cc ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                         "r"(v.w)
                         : "memory");
        }
    }
}

// ---------------------------------------------------------------- prep
// One warp per (row, head): Delta = sum_e dO * O in fp32, L2 = L * log2(e).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep(const __nv_bfloat16 *o, const __nv_bfloat16 *dout, const float *lse,
                                                float *delta, float *lse2, int n, int n_pad, int heads) {
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long items = (long long)n_pad * heads;
    if (warp >= items) return;
    const int h = (int)(warp / n_pad), r = (int)(warp % n_pad);
    float acc = 0.f;
    if (r < n) {
        constexpr int E = D / 32;     // 2 or 4 elements per lane, one 4- or 8-byte load
        using Vec = typename std::conditional<E == 4, uint2, uint32_t>::type;
        const Vec vo = *reinterpret_cast<const Vec *>(o + ((size_t)r * heads + h) * D + lane * E);
        const Vec vd = *reinterpret_cast<const Vec *>(dout + ((size_t)r * heads + h) * D + lane * E);
        const __nv_bfloat16 *eo = reinterpret_cast<const __nv_bfloat16 *>(&vo);
        const __nv_bfloat16 *ed = reinterpret_cast<const __nv_bfloat16 *>(&vd);
#pragma unroll
        for (int e = 0; e < E; ++e) acc = fmaf(__bfloat162float(eo[e]), __bfloat162float(ed[e]), acc);
    }
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (lane == 0) {
        delta[(size_t)h * n_pad + r] = acc;
        lse2[(size_t)h * n_pad + r] = r < n ? lse[(size_t)h * n + r] * kLog2e : INFINITY;
    }
}


// ---------------------------------------------------------------- dK, dV
// P^T and dS^T for 16 query columns of one key row (scores s[s0 .. s0+15]),
// written packed as bf16 pairs: p = exp2(s * sl2 - l2) (0 for columns below
// `lo`), ds = p * (dp - delta), with L*log2e and Delta of each column read
// from shared memory
// (broadcast: every thread reads the same column).  The arithmetic is in
// f32x2 pairs: scalar fp32 FMA, add and multiply instructions slow the
// tensor core of the SM down (by almost half, in a probe where one warp
// issues them beside an MMA loop), the paired forms hardly at all.
template <bool MASK>
__device__ __forceinline__ void pt_dst_piece(const uint32_t (&s)[32], int s0, const uint32_t (&dp)[16],
                                             const float *l2s, const float *dls, float sl2, int lo,
                                             uint32_t (&pk)[8], uint32_t (&dk)[8]) {
    const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
        const float4 l = *reinterpret_cast<const float4 *>(l2s + e);
        const float4 d = *reinterpret_cast<const float4 *>(dls + e);
        const float2 nl[2] = {make_float2(-l.x, -l.y), make_float2(-l.z, -l.w)};
        const float2 nd[2] = {make_float2(-d.x, -d.y), make_float2(-d.z, -d.w)};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int col = e + 2 * u;
            const float2 x =
                ffma2(make_float2(__uint_as_float(s[s0 + col]), __uint_as_float(s[s0 + col + 1])), sl2x2, nl[u]);
            float2 pr = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            if (MASK) {
                pr.x = col >= lo ? pr.x : 0.f;
                pr.y = col + 1 >= lo ? pr.y : 0.f;
            }
            const float2 g = fadd2(make_float2(__uint_as_float(dp[col]), __uint_as_float(dp[col + 1])), nd[u]);
            const float2 ds = fmul2(pr, g);
            pk[col / 2] = pack_bf16x2(pr.x, pr.y);
            dk[col / 2] = pack_bf16x2(ds.x, ds.y);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kDkdvThreads, 1) bwd_dkdv(const __grid_constant__ BwdParams p) {
    using L = DkdvLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sK = s_base + L::kA, sV = sK + L::kTile;
    auto stage_b = [&](int t) { return s_base + L::kB + (t & 1) * L::kStage; };   // Q, dO, L2[128], Delta[128]
    const uint32_t bars = s_base + L::kBars;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int n_kt = (p.n + kBT - 1) / kBT;
    const int kt = blockIdx.x / p.heads, head = blockIdx.x % p.heads;   // heaviest (kt = 0) first
    const int n_qt = n_kt;
    const int i_first = ((kt * kBT) / p.kpf) * p.kpf / kBT;            // first query tile that sees this key tile
    const int T = n_qt - i_first;

    if (threadIdx.x == 0) {
        mbar_init(bar(L::bA), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::bFull + s), 1);
            mbar_init(bar(L::bEmpty + s), 1);
        }
        mbar_init(bar(L::bS), 1);
        mbar_init(bar(L::bSread), 8);
        mbar_init(bar(L::bPh), 4);   // the softmax group of query columns 0-63
        mbar_init(bar(L::bP), 4);    // the group of columns 64-127
        mbar_init(bar(L::bO), 1);
        mbar_init(bar(L::bEpi), 2 * kBT);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // TMEM: S^T [0,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D).
    // Step t (query tile i_first + t): the softmax reads the whole S^T row
    // into registers first, so S^T(t+1) can be computed into [0,128) while
    // it works; P^T and dS^T of each 16-column group g go, packed, into the
    // dP^T columns [128+16g, 128+16g+16) the group has just read (P^T in
    // the first 8, dS^T in the last 8).  dV and dK of the first 64 query
    // columns start while the softmax does the other 64; dP^T(t+1) follows
    // the last of them.

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_tx(bar(L::bA), 2 * L::kTile);
            load_tile<D>(sK, &p.tm_k, bar(L::bA), head, kt * kBT);
            load_tile<D>(sV, &p.tm_v, bar(L::bA), head, kt * kBT);
            for (int t = 0; t < T; ++t) {
                const int st = t & 1, use = t >> 1;
                if (use > 0 && !mbar_wait(bar(L::bEmpty + st), (use - 1) & 1, kBwdWaitNs)) {
                    bwd_timeout(p, abort_flag);
                    break;
                }
                if (*abort_flag) break;
                const int i = i_first + t;
                const uint32_t sb = stage_b(t);
                mbar_arrive_tx(bar(L::bFull + st), 2 * L::kTile + 1024);
                load_tile<D>(sb, &p.tm_q, bar(L::bFull + st), head, i * kBT);
                load_tile<D>(sb + L::kTile, &p.tm_do, bar(L::bFull + st), head, i * kBT);
                bulk_load(sb + 2 * L::kTile, p.lse2 + (size_t)head * p.n_pad + i * kBT, 512, bar(L::bFull + st));
                bulk_load(sb + 2 * L::kTile + 512, p.delta + (size_t)head * p.n_pad + i * kBT, 512,
                          bar(L::bFull + st));
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBT, kBT, 0, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBT, D, 0, 1);
            const uint64_t descK = smem_desc_sw128(sK, 16, 1024), descV = smem_desc_sw128(sV, 16, 1024);
            auto full = [&](int t) {
                return mbar_wait(bar(L::bFull + (t & 1)), (t >> 1) & 1, kBwdWaitNs) && !*abort_flag;
            };
            // dV += P^T dO and dK += dS^T Q over query rows [64h, 64h+64) of step t
            auto dvdk_half = [&](int t, int h) {
                const uint32_t sb = stage_b(t);
#pragma unroll
                for (int kk = 0; kk < kHalf / 16; ++kk) {
                    const int q16 = h * (kHalf / 16) + kk;                       // 16-row group of queries
                    const uint32_t col = 128 + 16 * q16;                         // its packed P^T, then dS^T
                    const uint32_t acc = (t > 0 || q16 > 0) ? 1u : 0u;
                    const uint64_t rows = (uint64_t)((q16 * 2048) >> 4);
                    mma_ts(tmem + 256, tmem + col, smem_desc_sw128(sb + L::kTile, 16384, 1024) + rows, idesc_o, acc);
                    mma_ts(tmem + 256 + D, tmem + col + 8, smem_desc_sw128(sb, 16384, 1024) + rows, idesc_o, acc);
                }
            };
            bool ok = mbar_wait(bar(L::bA), 0, kBwdWaitNs) && full(0);
            if (ok) {
                tc_fence_after();
                mma_tile_ss<D>(tmem + 0, descK, smem_desc_sw128(stage_b(0), 16, 1024), idesc_s);              // S^T(0)
                mma_tile_ss<D>(tmem + 128, descV, smem_desc_sw128(stage_b(0) + L::kTile, 16, 1024), idesc_s); // dP^T(0)
                tc_commit(bar(L::bS));
            }
            for (int t = 0; ok && t < T; ++t) {
                ok = mbar_wait(bar(L::bSread), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                if (t + 1 < T) {
                    ok = full(t + 1);
                    if (!ok) break;
                    tc_fence_after();
                    mma_tile_ss<D>(tmem + 0, descK, smem_desc_sw128(stage_b(t + 1), 16, 1024), idesc_s);      // S^T(t+1)
                }
                ok = mbar_wait(bar(L::bPh), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                dvdk_half(t, 0);
                ok = mbar_wait(bar(L::bP), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                dvdk_half(t, 1);
                tc_commit(bar(L::bEmpty + (t & 1)));   // Q(t), dO(t) read by their last MMAs
                if (t + 1 < T) {
                    mma_tile_ss<D>(tmem + 128, descV, smem_desc_sw128(stage_b(t + 1) + L::kTile, 16, 1024),
                                   idesc_s);                                                               // dP^T(t+1)
                    tc_commit(bar(L::bS));
                }
            }
            if (!ok) bwd_timeout(p, abort_flag);
            tc_commit(bar(L::bO));   // all MMAs above done (also on the error path)
        }
        __syncwarp();
    } else if (warp >= 4) {
        const int sub = warp & 3;                          // TMEM lane quarter (warp id mod 4)
        const int grp = (warp - 4) >> 2;                   // query columns [64 grp, 64 grp + 64)
        const int row = sub * 32 + lane;
        const uint32_t lane_bits = (uint32_t)(sub * 32) << 16;
        const uint32_t tS = tmem + lane_bits + 64 * grp, tdP = tmem + lane_bits + 128 + 64 * grp;
        const int kr = kt * kBT + row;                     // key row
        const int q_lo = (kr / p.kpf) * p.kpf;             // first query row that sees it
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int i = i_first + t;
            const float *l2s =
                reinterpret_cast<const float *>(smem + L::kB + (t & 1) * L::kStage + 2 * L::kTile) + 64 * grp;
            const float *dls = l2s + kBT;
            bool w = !*abort_flag && mbar_wait(bar(L::bS), t & 1, kBwdWaitNs);
            w = __all_sync(0xffffffffu, w);
            if (!w) { ok = false; break; }
            tc_fence_after();
            uint32_t s0[32], s1[32], dpa[16], dpb[16];
            tmem_ld32(tS, s0);
            tmem_ld32(tS + 32, s1);
            tmem_ld16(tdP, dpa);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::bSread));   // S^T's columns are free for S^T(t+1)
            const int lo = q_lo - i * kBT - 64 * grp;      // columns below lo are hidden from this key
            // 16-column pieces of this warp's 64: piece h's dP^T loads while
            // piece h-1 is computed, and its P^T and dS^T (8 packed columns
            // each) go over its own 16 dP^T columns
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t(&cur)[16] = (h & 1) ? dpb : dpa;
                uint32_t(&nxt)[16] = (h & 1) ? dpa : dpb;
                if (h + 1 < 4) tmem_ld16(tdP + 16 * (h + 1), nxt);
                uint32_t pk[8], dk[8];
                if (__any_sync(0xffffffffu, lo - 16 * h > 0))   // warp-uniform: some column hidden
                    pt_dst_piece<true>(h < 2 ? s0 : s1, 16 * (h & 1), cur, l2s + 16 * h, dls + 16 * h,
                                       p.scale_log2, lo - 16 * h, pk, dk);
                else
                    pt_dst_piece<false>(h < 2 ? s0 : s1, 16 * (h & 1), cur, l2s + 16 * h, dls + 16 * h,
                                        p.scale_log2, 0, pk, dk);
                tmem_st8(tdP + 16 * h, pk);
                tmem_st8(tdP + 16 * h + 8, dk);
                if (h + 1 < 4) tmem_wait_ld_regs16(nxt);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(grp == 0 ? L::bPh : L::bP));
        }
        // epilogue: dV -> V's tile, dK * scale -> K's tile, then TMA stores
        bool w = ok && !*abort_flag && mbar_wait(bar(L::bO), 0, kBwdWaitNs);
        w = __all_sync(0xffffffffu, w);
        if (w) {
            tc_fence_after();
            if (grp == 0) acc_to_smem<D>(tmem + lane_bits + 256, 1.f, sV, row);
            else acc_to_smem<D>(tmem + lane_bits + 256 + D, p.scale, sK, row);
            fence_proxy_async_smem();
        }
        mbar_arrive(bar(L::bEpi));
        if (grp == 0 && row == 0) {
            const bool all = w && mbar_wait(bar(L::bEpi), 0, kBwdWaitNs);
            if (all) {
                for (int b = 0; b < D / 64; ++b) {
                    tma_store_3d(&p.tm_dv, sV + b * 16384, b * 64, head, kt * kBT);
                    tma_store_3d(&p.tm_dk, sK + b * 16384, b * 64, head, kt * kBT);
                }
                bulk_commit();
                bulk_wait_read0();
            } else {
                bwd_timeout(p, abort_flag);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- dQ
// dS for 32 key columns [32c, 32c+32) of one query row, packed as bf16
// pairs: p = exp2(s * sl2 - l2) (0 for columns at or past `hi`),
// ds = p * (dp - delta), dp from the row's registers; f32x2 arithmetic (see
// pt_dst_piece).
template <bool MASK>
__device__ __forceinline__ void ds_chunk(const uint32_t (&s)[32], const uint32_t (&dpr)[128], int c, float l2,
                                         float dl, float sl2, int hi, uint32_t (&dk)[16]) {
    const float2 sl2x2 = make_float2(sl2, sl2), nl2 = make_float2(-l2, -l2), ndl = make_float2(-dl, -dl);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float2 x = ffma2(make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sl2x2, nl2);
        float2 pr = make_float2(fast_exp2(x.x), fast_exp2(x.y));
        if (MASK) {
            pr.x = e < hi ? pr.x : 0.f;
            pr.y = e + 1 < hi ? pr.y : 0.f;
        }
        const float2 g =
            fadd2(make_float2(__uint_as_float(dpr[32 * c + e]), __uint_as_float(dpr[32 * c + e + 1])), ndl);
        const float2 ds = fmul2(pr, g);
        dk[e / 2] = pack_bf16x2(ds.x, ds.y);
    }
}

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1) bwd_dq(const __grid_constant__ BwdParams p) {
    using L = DqLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ = s_base + L::kA, sdO = sQ + L::kTile;
    auto k_slot = [&](int t) { return s_base + L::kK + (t % L::kKSlots) * L::kTile; };
    auto v_slot = [&](int t) { return s_base + L::kV + (t % L::kVSlots) * L::kTile; };
    const uint32_t bars = s_base + L::kBars;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int n_qt = (p.n + kBT - 1) / kBT;
    const int qt = n_qt - 1 - blockIdx.x / p.heads, head = blockIdx.x % p.heads;   // heaviest (last) first
    const int q_last = min(qt * kBT + kBT - 1, p.n - 1);
    const int vis_end = min(p.n, (q_last / p.kpf + 1) * p.kpf);   // keys the tile's last row sees
    const int T = (vis_end + kBT - 1) / kBT;

    if (threadIdx.x == 0) {
        mbar_init(bar(L::bA), 1);
        for (int s = 0; s < L::kKSlots; ++s) {
            mbar_init(bar(L::bKFull + s), 1);
            mbar_init(bar(L::bKEmpty + s), 1);
        }
        for (int s = 0; s < L::kVSlots; ++s) {
            mbar_init(bar(L::bVFull + s), 1);
            mbar_init(bar(L::bVEmpty + s), 1);
        }
        mbar_init(bar(L::bS), 1);
        mbar_init(bar(L::bDPread), 4);
        mbar_init(bar(L::bPh), 4);
        mbar_init(bar(L::bP), 4);
        mbar_init(bar(L::bO), 1);
        mbar_init(bar(L::bEpi), kBT);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // TMEM: S buffers [0,128), [128,256) (key tile t in buffer t % 2; its dS
    // is written, packed, over the first 16 of each 32-column group of S it
    // came from); dP [256,384); dQ [384,384+D).  The softmax reads the whole
    // dP row into registers first, so dP(t+1) is computed while it works.
    // dQ of the first 64 keys starts while the softmax does the other 64.

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_tx(bar(L::bA), 2 * L::kTile);
            load_tile<D>(sQ, &p.tm_q, bar(L::bA), head, qt * kBT);
            load_tile<D>(sdO, &p.tm_do, bar(L::bA), head, qt * kBT);
            for (int t = 0; t < T; ++t) {
                const int ks = t % L::kKSlots, ku = t / L::kKSlots;
                if (ku > 0 && !mbar_wait(bar(L::bKEmpty + ks), (ku - 1) & 1, kBwdWaitNs)) {
                    bwd_timeout(p, abort_flag);
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_tx(bar(L::bKFull + ks), L::kTile);
                load_tile<D>(k_slot(t), &p.tm_k, bar(L::bKFull + ks), head, t * kBT);
                const int vs = t % L::kVSlots, vu = t / L::kVSlots;
                if (vu > 0 && !mbar_wait(bar(L::bVEmpty + vs), (vu - 1) & 1, kBwdWaitNs)) {
                    bwd_timeout(p, abort_flag);
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_tx(bar(L::bVFull + vs), L::kTile);
                load_tile<D>(v_slot(t), &p.tm_v, bar(L::bVFull + vs), head, t * kBT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBT, kBT, 0, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBT, D, 0, 1);
            const uint64_t descQ = smem_desc_sw128(sQ, 16, 1024), descdO = smem_desc_sw128(sdO, 16, 1024);
            auto k_full = [&](int t) {
                return mbar_wait(bar(L::bKFull + t % L::kKSlots), (t / L::kKSlots) & 1, kBwdWaitNs) && !*abort_flag;
            };
            auto v_full = [&](int t) {
                return mbar_wait(bar(L::bVFull + t % L::kVSlots), (t / L::kVSlots) & 1, kBwdWaitNs) && !*abort_flag;
            };
            // dQ += dS K over keys [64h, 64h+64) of tile t
            auto dq_half = [&](int t, int h) {
                const uint32_t buf = 128 * (t & 1);
#pragma unroll
                for (int kk = 0; kk < kHalf / 16; ++kk) {
                    const int k16 = h * (kHalf / 16) + kk;                       // 16-key group
                    const uint32_t col = buf + 32 * (k16 >> 1) + 8 * (k16 & 1);  // its packed dS columns
                    mma_ts(tmem + 384, tmem + col,
                           smem_desc_sw128(k_slot(t), 16384, 1024) + (uint64_t)((k16 * 2048) >> 4), idesc_o,
                           (t > 0 || k16 > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(bar(L::bA), 0, kBwdWaitNs) && k_full(0) && v_full(0);
            if (ok) {
                tc_fence_after();
                mma_tile_ss<D>(tmem + 0, descQ, smem_desc_sw128(k_slot(0), 16, 1024), idesc_s);     // S(0)
                mma_tile_ss<D>(tmem + 256, descdO, smem_desc_sw128(v_slot(0), 16, 1024), idesc_s);  // dP(0)
                tc_commit(bar(L::bS));
                tc_commit(bar(L::bVEmpty + 0));
            }
            // Per step: dP(t+1) once the softmax holds dP(t), dQ of the first
            // 64 keys, then S(t+1): K(t+1) reuses the slot of K(t-2), freed
            // by the last dQ MMA two steps back, and issuing S(t+1) this late
            // gives its load time to land.
            for (int t = 0; ok && t < T; ++t) {
                ok = mbar_wait(bar(L::bDPread), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                if (t + 1 < T) {
                    ok = v_full(t + 1);
                    if (!ok) break;
                    tc_fence_after();
                    mma_tile_ss<D>(tmem + 256, descdO, smem_desc_sw128(v_slot(t + 1), 16, 1024), idesc_s);  // dP(t+1)
                    tc_commit(bar(L::bVEmpty + (t + 1) % L::kVSlots));
                }
                ok = mbar_wait(bar(L::bPh), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                dq_half(t, 0);
                if (t + 1 < T) {
                    ok = k_full(t + 1);
                    if (!ok) break;
                    tc_fence_after();
                    mma_tile_ss<D>(tmem + 128 * ((t + 1) & 1), descQ, smem_desc_sw128(k_slot(t + 1), 16, 1024),
                                   idesc_s);                                                          // S(t+1)
                    tc_commit(bar(L::bS));   // S(t+1) and dP(t+1) done
                }
                ok = mbar_wait(bar(L::bP), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                dq_half(t, 1);
                tc_commit(bar(L::bKEmpty + t % L::kKSlots));
            }
            if (!ok) bwd_timeout(p, abort_flag);
            tc_commit(bar(L::bO));
        }
        __syncwarp();
    } else if (warp >= 4) {
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const uint32_t lane_bits = (uint32_t)(sub * 32) << 16;
        const uint32_t tdP = tmem + lane_bits + 256;
        const int qr = qt * kBT + row;                                  // query row
        const int row_end = min(p.n, (qr / p.kpf + 1) * p.kpf);        // keys it sees: [0, row_end)
        const float l2v = p.lse2[(size_t)head * p.n_pad + qr];          // +inf past n: P = 0
        const float dlv = p.delta[(size_t)head * p.n_pad + qr];
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            bool w = !*abort_flag && mbar_wait(bar(L::bS), t & 1, kBwdWaitNs);
            w = __all_sync(0xffffffffu, w);
            if (!w) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = tmem + lane_bits + 128 * (t & 1);
            uint32_t dpr[128], sv0[32], sv1[32];
            tmem_ld128(tdP, dpr);
            tmem_ld32(tS, sv0);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::bDPread));   // dP's columns are free for dP(t+1)
            const int hi = row_end - t * kBT;                           // columns at and past hi are hidden
            // S group c+1 loads while group c is computed
#pragma unroll   // constant c: the dP row stays in registers
            for (int c = 0; c < 4; ++c) {
                uint32_t(&cur)[32] = (c & 1) ? sv1 : sv0;
                uint32_t(&nxt)[32] = (c & 1) ? sv0 : sv1;
                if (c + 1 < 4) tmem_ld32(tS + 32 * (c + 1), nxt);
                uint32_t dk[16];
                if (__any_sync(0xffffffffu, hi - 32 * c < 32))   // warp-uniform: some column hidden
                    ds_chunk<true>(cur, dpr, c, l2v, dlv, p.scale_log2, hi - 32 * c, dk);
                else
                    ds_chunk<false>(cur, dpr, c, l2v, dlv, p.scale_log2, 32, dk);
                tmem_st16(tS + 32 * c, dk);
                if (c == 1 || c == 3) {
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(c == 1 ? L::bPh : L::bP));
                }
                if (c + 1 < 4) tmem_wait_ld_regs(nxt);
            }
        }
        bool w = ok && !*abort_flag && mbar_wait(bar(L::bO), 0, kBwdWaitNs);
        w = __all_sync(0xffffffffu, w);
        if (w) {
            tc_fence_after();
            acc_to_smem<D>(tmem + lane_bits + 384, p.scale, sQ, row);   // Q's tile is free after the last MMA
            fence_proxy_async_smem();
        }
        mbar_arrive(bar(L::bEpi));
        if (row == 0) {
            const bool all = w && mbar_wait(bar(L::bEpi), 0, kBwdWaitNs);
            if (all) {
                for (int b = 0; b < D / 64; ++b) tma_store_3d(&p.tm_dq, sQ + b * 16384, b * 64, head, qt * kBT);
                bulk_commit();
                bulk_wait_read0();
            } else {
                bwd_timeout(p, abort_flag);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_bwd_t(const BwdParams &bp, const BwdProblem &pb, cudaStream_t s) {
    using L = DkdvLayout<D>;
    static std::atomic<unsigned long long> configured{0};   // one bit per device (0..63)
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        cudaError_t e = cudaFuncSetAttribute(bwd_dkdv<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(bwd_dq<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DqLayout<D>::kAlloc);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_release);
    }
    const long long prep_warps = (long long)bp.n_pad * bp.heads;
    bwd_prep<D><<<(unsigned)((prep_warps * 32 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(pb.o), static_cast<const __nv_bfloat16 *>(pb.dout), pb.lse,
        const_cast<float *>(bp.delta), const_cast<float *>(bp.lse2), bp.n, bp.n_pad, bp.heads);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    const unsigned tiles = (unsigned)((bp.n + kBT - 1) / kBT) * (unsigned)bp.heads;
    bwd_dkdv<D><<<tiles, kDkdvThreads, L::kAlloc, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    bwd_dq<D><<<tiles, kDqThreads, DqLayout<D>::kAlloc, s>>>(bp);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

size_t bwd_scratch_bytes(int n, int heads) {
    const size_t n_pad = ((size_t)n + kBT - 1) / kBT * kBT;
    return 2 * (size_t)heads * n_pad * sizeof(float);
}

cudaError_t launch_attn_bwd(const BwdProblem &pb, unsigned *status, void *scratch, cudaStream_t s) {
    BwdParams bp;
    memset(&bp, 0, sizeof(bp));
    const uint64_t D = (uint64_t)pb.head_dim;
    const uint64_t H = (uint64_t)pb.heads, N = (uint64_t)pb.n;
    if (!make_tmap_bf16(&bp.tm_q, pb.q, D, H, N, 1, kBT) || !make_tmap_bf16(&bp.tm_k, pb.k, D, H, N, 1, kBT) ||
        !make_tmap_bf16(&bp.tm_v, pb.v, D, H, N, 1, kBT) || !make_tmap_bf16(&bp.tm_do, pb.dout, D, H, N, 1, kBT) ||
        !make_tmap_bf16(&bp.tm_dq, pb.dq, D, H, N, 1, kBT) || !make_tmap_bf16(&bp.tm_dk, pb.dk, D, H, N, 1, kBT) ||
        !make_tmap_bf16(&bp.tm_dv, pb.dv, D, H, N, 1, kBT))
        return cudaErrorInvalidValue;
    bp.n = pb.n;
    bp.n_pad = (pb.n + kBT - 1) / kBT * kBT;
    bp.heads = pb.heads;
    bp.kpf = pb.kpf;
    bp.scale = pb.scale;
    bp.scale_log2 = pb.scale * kLog2e;
    bp.status = status;
    float *f = static_cast<float *>(scratch);
    bp.delta = f;
    bp.lse2 = f + (size_t)pb.heads * bp.n_pad;
    if (pb.head_dim == 128) return launch_bwd_t<128>(bp, pb, s);
    if (pb.head_dim == 64) return launch_bwd_t<64>(bp, pb, s);
    return cudaErrorInvalidValue;
}

}  // namespace rtr
