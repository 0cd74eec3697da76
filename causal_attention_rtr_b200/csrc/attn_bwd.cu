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
//               key tile's first frame), each as two halves of 64 queries.
//               Per half: S^T = K Q^T and dP^T = V dO^T into one of two TMEM
//               buffers, the softmax warps turn them into P^T and dS^T (bf16,
//               back into TMEM), then dV += P^T dO and dK += dS^T Q with the
//               "A in tensor memory" form; the tensor core runs the other
//               buffer's MMAs meanwhile.
//   bwd_dq      query-stationary: one CTA per (head, 128-query tile); streams
//               the key tiles it sees.  S = Q K^T and dP = dO V^T into TMEM,
//               dS (bf16) back into TMEM, dQ += dS K.  S has two TMEM
//               buffers, so S of the next key tile runs during this tile's
//               softmax; dP has one (dS lives in it until dQ has read it).
//               (bwd_dkdv's half-tile scheme measured 14 % slower here: its
//               64-wide S and dP MMAs re-read Q and dO per half, and each
//               half pays the softmax hand-off again.)
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
constexpr int kBwdThreads = 256;
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

// Shared-memory layout of both main kernels: two stationary tiles A0, A1
// (dkdv: K, V; dq: Q, dO), two stages of two streamed tiles B0, B1 (dkdv: Q,
// dO; dq: K, V) plus, per stage, 128 floats each of L*log2e and Delta
// (dkdv only), then the barriers.
template <int D>
struct BwdLayout {
    static constexpr int kTile = kBT * D * 2;
    static constexpr int kA = 0;                         // A0, A1
    static constexpr int kStage = 2 * kTile + 1024;      // B0, B1, row stats
    static constexpr int kB = 2 * kTile;                 // stage s at kB + s * kStage
    static constexpr int kBars = kB + 2 * kStage;
    static constexpr int bA = 0, bFull = 1, bEmpty = 3, bS = 5, bP = 7, bO = 9, bEpi = 10, kNumBars = 11;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

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

// TS MMA chain over KR rows of B: C[128 x D] (+)= A[128 x KR] B[KR x D] with
// A packed bf16 pairs in TMEM at a_tmem (8 columns per 16 rows of B) and B
// read as MN-major from the TMA layout (16 rows = 2048 bytes per step).
template <int D, int KR>
__device__ __forceinline__ void mma_tile_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                            bool acc) {
#pragma unroll
    for (int kk = 0; kk < KR / 16; ++kk)
        mma_ts(d_tmem, a_tmem + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4), idesc, (acc || kk > 0) ? 1u : 0u);
}

constexpr int kHalf = 64;     // rows of the streamed half tile (MMA N of S / dP)

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

// Packed P / dS for 32 columns of one row: p = exp2(s * sl2 - l2) (0 where
// masked), ds = p * (dp - delta).  `l2`, `dl` are per column (dkdv) or
// broadcast scalars (dq), chosen by the caller through the arrays.
__device__ __forceinline__ void p_ds_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], const float (&l2)[32],
                                           const float (&dl)[32], float sl2, int lo, int hi, uint32_t (&pk)[16],
                                           uint32_t (&dk)[16]) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float p0 = fast_exp2(fmaf(__uint_as_float(s[e]), sl2, -l2[e]));
        float p1 = fast_exp2(fmaf(__uint_as_float(s[e + 1]), sl2, -l2[e + 1]));
        p0 = (e >= lo && e < hi) ? p0 : 0.f;
        p1 = (e + 1 >= lo && e + 1 < hi) ? p1 : 0.f;
        pk[e / 2] = pack_bf16x2(p0, p1);
        dk[e / 2] = pack_bf16x2(p0 * (__uint_as_float(dp[e]) - dl[e]), p1 * (__uint_as_float(dp[e + 1]) - dl[e + 1]));
    }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkdv(const __grid_constant__ BwdParams p) {
    using L = BwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sK = s_base + L::kA, sV = sK + L::kTile;
    auto stage_b = [&](int st) { return s_base + L::kB + st * L::kStage; };   // Q, dO, L2[128], Delta[128]
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(L::bS + b), 1);
            mbar_init(bar(L::bP + b), 4);
        }
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
    // TMEM: S^T / P^T buffers [0,64), [64,128); dP^T / dS^T buffers [128,192),
    // [192,256); dV [256,256+D); dK [256+D,256+2D).  Each streamed query tile
    // is taken as two halves of 64 queries (step t: tile t/2, half t%2,
    // buffer t%2): while the softmax works on step t the tensor core runs
    // dV/dK of step t-1 and S^T/dP^T of step t+1.

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
                const uint32_t sb = stage_b(st);
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
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBT, D, 0, 1);
            const uint64_t descK = smem_desc_sw128(sK, 16, 1024), descV = smem_desc_sw128(sV, 16, 1024);
            constexpr uint32_t idesc_h = idesc_bf16_f32(kBT, kHalf, 0, 0);
            bool ok = mbar_wait(bar(L::bA), 0, kBwdWaitNs);
            for (int t = 0; ok && t <= 2 * T; ++t) {
                if (t < 2 * T) {
                    const int ti = t >> 1, h = t & 1, b = t & 1;
                    const uint32_t sb = stage_b(ti & 1);
                    if (h == 0) {
                        ok = mbar_wait(bar(L::bFull + (ti & 1)), (ti >> 1) & 1, kBwdWaitNs) && !*abort_flag;
                        if (!ok) break;
                    }
                    tc_fence_after();
                    const uint32_t hoff = (uint32_t)(h * kHalf * 128);
                    mma_tile_ss<D>(tmem + 64 * b, descK, smem_desc_sw128(sb + hoff, 16, 1024), idesc_h);   // S^T
                    mma_tile_ss<D>(tmem + 128 + 64 * b, descV, smem_desc_sw128(sb + L::kTile + hoff, 16, 1024),
                                   idesc_h);                                                           // dP^T
                    tc_commit(bar(L::bS + b));
                }
                if (t >= 1) {
                    const int tp = t - 1, ti = tp >> 1, h = tp & 1, b = tp & 1;
                    const uint32_t sb = stage_b(ti & 1);
                    ok = mbar_wait(bar(L::bP + b), (tp >> 1) & 1, kBwdWaitNs) && !*abort_flag;
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t hoff = (uint32_t)(h * kHalf * 128);
                    mma_tile_ts<D, kHalf>(tmem + 256, tmem + 64 * b, smem_desc_sw128(sb + L::kTile + hoff, 16384, 1024),
                                          idesc_o, tp > 0);                                    // dV += P^T dO
                    mma_tile_ts<D, kHalf>(tmem + 256 + D, tmem + 128 + 64 * b, smem_desc_sw128(sb + hoff, 16384, 1024),
                                          idesc_o, tp > 0);                                    // dK += dS^T Q
                    if (h == 1) tc_commit(bar(L::bEmpty + (ti & 1)));
                }
            }
            if (!ok) bwd_timeout(p, abort_flag);
            tc_commit(bar(L::bO));   // all MMAs above done (also on the error path)
        }
        __syncwarp();
    } else if (warp >= 4) {
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const uint32_t lane_bits = (uint32_t)(sub * 32) << 16;
        const int kr = kt * kBT + row;                     // key row
        const int q_lo = (kr / p.kpf) * p.kpf;             // first query row that sees it
        bool ok = true;
        for (int t = 0; t < 2 * T; ++t) {
            const int ti = t >> 1, h = t & 1, b = t & 1;
            const int i = i_first + ti;
            const float *l2s =
                reinterpret_cast<const float *>(smem + L::kB + (ti & 1) * L::kStage + 2 * L::kTile) + h * kHalf;
            const float *dls = l2s + 128;
            const uint32_t tS = tmem + lane_bits + 64 * b, tdP = tS + 128;
            bool w = !*abort_flag && mbar_wait(bar(L::bS + b), (t >> 1) & 1, kBwdWaitNs);
            w = __all_sync(0xffffffffu, w);
            if (!w) { ok = false; break; }
            tc_fence_after();
            const int lo = q_lo - i * kBT - h * kHalf;     // columns below lo are hidden from this key
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t s[32], dp[32], pk[16], dk[16];
                float l2[32], dl[32];
                tmem_ld32(tS + 32 * c, s);
                tmem_ld32(tdP + 32 * c, dp);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(l2s + 32 * c + e);
                    const float4 bq = *reinterpret_cast<const float4 *>(dls + 32 * c + e);
                    l2[e] = a.x; l2[e + 1] = a.y; l2[e + 2] = a.z; l2[e + 3] = a.w;
                    dl[e] = bq.x; dl[e + 1] = bq.y; dl[e + 2] = bq.z; dl[e + 3] = bq.w;
                }
                tmem_wait_ld();
                p_ds_chunk(s, dp, l2, dl, p.scale_log2, lo - 32 * c, 32, pk, dk);
                tmem_st16(tS + 16 * c, pk);
                tmem_st16(tdP + 16 * c, dk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::bP + b));
        }
        // epilogue: dV -> V's tile, dK * scale -> K's tile, then TMA stores
        bool w = ok && !*abort_flag && mbar_wait(bar(L::bO), 0, kBwdWaitNs);
        w = __all_sync(0xffffffffu, w);
        if (w) {
            tc_fence_after();
            acc_to_smem<D>(tmem + lane_bits + 256, 1.f, sV, row);
            acc_to_smem<D>(tmem + lane_bits + 256 + D, p.scale, sK, row);
            fence_proxy_async_smem();
        }
        mbar_arrive(bar(L::bEpi));
        if (row == 0) {
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
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq(const __grid_constant__ BwdParams p) {
    using L = BwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ = s_base + L::kA, sdO = sQ + L::kTile;
    auto stage_b = [&](int st) { return s_base + L::kB + st * L::kStage; };   // K, V
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
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::bFull + s), 1);
            mbar_init(bar(L::bEmpty + s), 1);
        }
        mbar_init(bar(L::bS), 1);   // one S / dP buffer: bS + 0, bP + 0
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
    // TMEM: S buffers [0,128), [128,256) (tile t in buffer t % 2); dP / dS
    // [256,384); dQ [384,384+D).

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_tx(bar(L::bA), 2 * L::kTile);
            load_tile<D>(sQ, &p.tm_q, bar(L::bA), head, qt * kBT);
            load_tile<D>(sdO, &p.tm_do, bar(L::bA), head, qt * kBT);
            for (int t = 0; t < T; ++t) {
                const int st = t & 1, use = t >> 1;
                if (use > 0 && !mbar_wait(bar(L::bEmpty + st), (use - 1) & 1, kBwdWaitNs)) {
                    bwd_timeout(p, abort_flag);
                    break;
                }
                if (*abort_flag) break;
                const uint32_t sb = stage_b(st);
                mbar_arrive_tx(bar(L::bFull + st), 2 * L::kTile);
                load_tile<D>(sb, &p.tm_k, bar(L::bFull + st), head, t * kBT);
                load_tile<D>(sb + L::kTile, &p.tm_v, bar(L::bFull + st), head, t * kBT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBT, kBT, 0, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBT, D, 0, 1);
            const uint64_t descQ = smem_desc_sw128(sQ, 16, 1024), descdO = smem_desc_sw128(sdO, 16, 1024);
            // S(t+1) goes into the other S buffer while the softmax works on
            // tile t; dP(t+1) follows dQ(t), which reads dS(t) from dP's columns.
            bool ok = mbar_wait(bar(L::bA), 0, kBwdWaitNs) &&
                      mbar_wait(bar(L::bFull + 0), 0, kBwdWaitNs) && !*abort_flag;
            if (ok) {
                tc_fence_after();
                mma_tile_ss<D>(tmem + 0, descQ, smem_desc_sw128(stage_b(0), 16, 1024), idesc_s);                  // S(0)
                mma_tile_ss<D>(tmem + 256, descdO, smem_desc_sw128(stage_b(0) + L::kTile, 16, 1024), idesc_s);   // dP(0)
                tc_commit(bar(L::bS));
            }
            for (int t = 0; ok && t < T; ++t) {
                const int st = t & 1, stn = st ^ 1;
                const uint32_t sb = stage_b(st), sbn = stage_b(stn);
                if (t + 1 < T) {
                    ok = mbar_wait(bar(L::bFull + stn), ((t + 1) >> 1) & 1, kBwdWaitNs) && !*abort_flag;
                    if (!ok) break;
                    tc_fence_after();
                    mma_tile_ss<D>(tmem + 128 * ((t + 1) & 1), descQ, smem_desc_sw128(sbn, 16, 1024), idesc_s);  // S(t+1)
                }
                ok = mbar_wait(bar(L::bP), t & 1, kBwdWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                mma_tile_ts<D, kBT>(tmem + 384, tmem + 256, smem_desc_sw128(sb, 16384, 1024), idesc_o, t > 0);  // dQ += dS K
                tc_commit(bar(L::bEmpty + st));
                if (t + 1 < T) {
                    mma_tile_ss<D>(tmem + 256, descdO, smem_desc_sw128(sbn + L::kTile, 16, 1024), idesc_s);      // dP(t+1)
                    tc_commit(bar(L::bS));
                }
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
        float l2[32], dl[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            l2[e] = l2v;
            dl[e] = dlv;
        }
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            bool w = !*abort_flag && mbar_wait(bar(L::bS), t & 1, kBwdWaitNs);
            w = __all_sync(0xffffffffu, w);
            if (!w) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = tmem + lane_bits + 128 * (t & 1);
            const int hi = row_end - t * kBT;                           // columns at and past hi are hidden
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t s[32], dp[32], pk[16], dk[16];
                tmem_ld32(tS + 32 * c, s);
                tmem_ld32(tdP + 32 * c, dp);
                tmem_wait_ld();
                p_ds_chunk(s, dp, l2, dl, p.scale_log2, 0, hi - 32 * c, pk, dk);
                tmem_st16(tdP + 16 * c, dk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::bP));
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
    using L = BwdLayout<D>;
    static std::atomic<unsigned long long> configured{0};   // one bit per device (0..63)
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        cudaError_t e = cudaFuncSetAttribute(bwd_dkdv<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(bwd_dq<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
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
    bwd_dkdv<D><<<tiles, kBwdThreads, L::kAlloc, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    bwd_dq<D><<<tiles, kBwdThreads, L::kAlloc, s>>>(bp);
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
