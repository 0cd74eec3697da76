// gemm_tc.cu -- the projections of the DiT block on the 5th-generation
// tensor cores (sm_100a), each with its elementwise epilogue fused into the
// output stage.
//
// C = A W with A bf16 [m][k] (token-major activations) and W bf16 [k][n]
// (weights stored [in][out]), fp32 accumulation in tensor memory, then one
// of four epilogues applied to the fp32 tile before anything reaches global
// memory:
//   bias            out = bf16(C + b)
//   bias + GELU     out = bf16(GELU_tanh(C + b))
//   gated residual  x   = bf16(x + g (C + b))   (x updated in place; g = 1 if null)
//   QKV + rotary    q, k, v = bf16 of (C + b) split in thirds, q and k turned
//                   by the 3D rotary encoding of each token
// Every stored value is rounded once, from the same fp32 quantities a
// separate epilogue kernel would read back (papernotes.org note "DiT as
// Real-Time Rerenderer", Method > Overall Architecture: the DiT blocks around
// the frame-causal attention; the rotary form is RoFormer's, eq. 13-15, split
// over (frame, row, column) channel parts).
//
// Persistent kernel, one CTA per SM, 320 threads:
//   warp 0      TMA producer: per 64-wide K block, the A tile (128 rows x 64)
//               and the W tile (64 x BN, BN/64 boxes) into a ring of stages
//   warp 1      TMEM allocation and the tcgen05.mma issuer (one thread):
//               D[128 x BN] += A[128 x 16] W[16 x BN], A K-major and W
//               MN-major from 128-byte-swizzled shared memory
//   warps 2-9   epilogue: two warps per TMEM lane quarter (one thread per
//               row), each taking alternate 32-column chunks of the tile;
//               its arithmetic is in f32x2 pairs and the special-function
//               unit (scalar fp32 instructions slow the next tile's MMAs),
//               the rotary angles come from a table each CTA fills once
// A tile is 128 rows by BN = 128, 192 or 256 columns, or 256 by 256 (two
// 128-row sub-tiles whose MMAs share each stage of W).  When a tile's
// accumulators take at most 256 TMEM columns there are two buffers, so the
// epilogue of one tile overlaps the MMAs of the next; a 256 x 256 tile fills
// TMEM and waits for its epilogue.  Tiles are numbered with N fastest and
// dealt round-robin; the host picks the shape with a cost model (pick_tile).
// Operands come by TMA boxes from row-major memory, or as whole stages by
// one bulk copy from the packed layouts (dit_internal.h).  Every wait is bounded (1 s); a timeout latches RTR_E_TIMEOUT in the
// device status word and every role stops.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "dit_internal.h"
#include "internal.h"
#include "ptx.cuh"

namespace rtr {
namespace {

constexpr int kBM = 128;               // rows per tile
constexpr int kBK = 64;                // K per stage (one 128-byte swizzle row of bf16)
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kATileBytes = kBM * kBK * 2;          // 16 KB
constexpr int kBBoxBytes = kBK * 64 * 2;            // 8 KB: 64 K rows x 64 N columns
constexpr int kMaxSmem = 200 * 1024;                // stages share this
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr float kLog2RopeBase = 13.287712379549449f;   // log2(10000)
constexpr int kRopeTabMax = 2048;                       // table entries (float2) at most: 16 KB

struct GemmParams {
    CUtensorMap tm_a;   // A [m][k]: dims (k, m, 1), box (64, 128, 1)
    CUtensorMap tm_w;   // W [k][n]: dims (n, k, 1), box (64, 64, 1)
    const char *a_pk;   // packed A (a_packed) or null
    const char *w_pk;   // packed B (w_packed) or null
    int kb_total, nb_total;   // k / 64, n / 64 of the packed layouts
    int out_packed;     // bias / GELU output written in the packed A layout of [m][n]
    int m, n, k;
    int bn, n_tiles_n, n_tiles, k_blocks, stages;
    int msub;           // 128-row sub-tiles per tile (1 or 2): tiles of 128 * msub rows share each W stage
    int nbuf;           // accumulator buffers in TMEM (2 when msub * bn <= 256, else 1)
    const __nv_bfloat16 *bias, *gate;
    __nv_bfloat16 *out;                 // bias / GELU: [m][n]; gated residual: [m][n] in place
    __nv_bfloat16 *q, *kk, *v;          // QKV: [m][D] each, D = n / 3
    int D, head_dim, kpf, grid_w, t0, rope_dt, rope_dp;
    // rotary table in shared memory: (cos, sin) per (frame, time pair), then
    // per (row, row pair) and per (column, column pair); 0 entries: the
    // epilogue computes each angle itself
    int rope_entries, rope_frames, rope_rows;
    unsigned *status;
};

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&b);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

// GELU, tanh form, for a pair: 0.5 x (1 + tanh(y)) = x sigmoid(2y) =
// x / (1 + 2^(-2 y log2 e)), y = sqrt(2/pi) (x + 0.044715 x^3).  The pair
// arithmetic is f32x2 and the exponential and reciprocal are the special
// function unit's: scalar fp32 instructions in the epilogue would slow the
// next tile's MMAs down.  The sigmoid form has no cancellation; relative
// error about 1e-6, far below a bf16 step.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 gelu_tanh2(float2 x) {
    const float kC = -2.0f * 0.7978845608028654f * 1.4426950408889634f;   // -2 sqrt(2/pi) log2(e)
    const float2 v = ffma2(fmul2(x, x), make_float2(0.044715f, 0.044715f), make_float2(1.f, 1.f));
    const float2 z = fmul2(fmul2(x, v), make_float2(kC, kC));
    const float2 d = fadd2(make_float2(fast_exp2(z.x), fast_exp2(z.y)), make_float2(1.f, 1.f));
    return fmul2(x, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// Angle of rotary channel pair j of a section with `size` channels at
// position pos, as (cos, sin).
__device__ __forceinline__ float2 rope_angle(int j, int size, int pos) {
    const float theta = exp2f(-(float)(2 * j) / (float)size * kLog2RopeBase);
    float sn, cs;
    sincosf((float)pos * theta, &sn, &cs);
    return make_float2(cs, sn);
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

// The same with cluster-scope acquire, for barriers the peer CTA of a pair
// signals (its commits and its epilogue's releases).
__device__ __forceinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

__device__ __forceinline__ void raise_timeout(const GemmParams &p, volatile int *abort_flag) {
    *abort_flag = 1;
    atomicExch(p.status, (unsigned)RTR_E_TIMEOUT);
}

// The global inputs of one 32-column chunk of a row: bias (all epilogues),
// and for the gated residual the residual x and the gate.  They are loaded
// together, before the chunk's accumulators arrive from TMEM and before any
// of the chunk's stores, so their latencies overlap (loads issued one
// 8-column group at a time, each after the previous group's store, paid a
// DRAM round trip per group and made the epilogue, not the MMAs, bound the
// projection).
struct EpiIn {
    uint4 b[4], x[4], g[4];
};

__device__ __forceinline__ uint4 ld_nc(const __nv_bfloat16 *ptr) {
    return __ldg(reinterpret_cast<const uint4 *>(ptr));
}

template <int EPI>
__device__ __forceinline__ void epi_load(const GemmParams &p, long long row, int col, int nvalid, EpiIn &in) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        if (8 * g >= nvalid) break;
        in.b[g] = ld_nc(p.bias + col + 8 * g);
        if (EPI == kEpiGatedResidual) {
            in.x[g] = *reinterpret_cast<const uint4 *>(p.out + row * p.n + col + 8 * g);
            if (p.gate != nullptr) in.g[g] = ld_nc(p.gate + col + 8 * g);
        }
    }
}

// The epilogue of 32 consecutive accumulator columns [col, col + 32) of one
// row (nvalid of them inside the matrix, a multiple of 8), in f32x2 pairs,
// from the chunk's inputs `in`.  `rope` is the shared-memory rotary table
// (null: angles computed here).
template <int EPI>
__device__ __forceinline__ void epi_chunk(const GemmParams &p, const uint32_t (&acc)[32], const EpiIn &in,
                                          long long row, int col, int nvalid, int f_pos, int y_pos, int x_pos,
                                          const float2 *rope) {
    if (EPI == kEpiQkvRope) {
        const int part = col / p.D, cc = col - part * p.D;
        __nv_bfloat16 *dst = (part == 0 ? p.q : part == 1 ? p.kk : p.v) + row * p.D + cc;
        const int c0 = cc % p.head_dim;                 // channel of the first column within its head
        const int nt = p.rope_dt / 2, nd = p.rope_dp / 2;
        // the chunk's 16 (cos, sin) pairs first, all table reads issued before
        // any is used: channel pair c / 2 lies in the time, row or column
        // section, each indexed by the token's frame, row or column
        float2 cs[16];
        if (part < 2) {
            const int t_base = (f_pos - p.t0) * nt, y_base = p.rope_frames * nt + y_pos * nd - p.rope_dt / 2,
                      x_base = p.rope_frames * nt + (p.rope_rows + x_pos) * nd - (p.rope_dt + p.rope_dp) / 2;
#pragma unroll
            for (int pr = 0; pr < 16; ++pr) {
                if (2 * pr >= nvalid) break;
                const int c = c0 + 2 * pr, h = c / 2;
                if (rope != nullptr) {
                    const int idx = c < p.rope_dt ? t_base + h : c < p.rope_dt + p.rope_dp ? y_base + h : x_base + h;
                    cs[pr] = rope[idx];
                } else if (c < p.rope_dt) {
                    cs[pr] = rope_angle(h, p.rope_dt, f_pos);
                } else if (c < p.rope_dt + p.rope_dp) {
                    cs[pr] = rope_angle(h - p.rope_dt / 2, p.rope_dp, y_pos);
                } else {
                    cs[pr] = rope_angle(h - (p.rope_dt + p.rope_dp) / 2, p.rope_dp, x_pos);
                }
            }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (8 * g >= nvalid) break;
            float b[8], r[8];
            unpack8(in.b[g], b);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                float2 v = fadd2(make_float2(__uint_as_float(acc[8 * g + e]), __uint_as_float(acc[8 * g + e + 1])),
                                 make_float2(b[e], b[e + 1]));
                if (part < 2) {
                    const float2 t = cs[4 * g + e / 2];
                    // (a0 cos - a1 sin, a1 cos + a0 sin)
                    v = ffma2(v, make_float2(t.x, t.x), fmul2(make_float2(v.y, v.x), make_float2(-t.y, t.y)));
                }
                r[e] = v.x;
                r[e + 1] = v.y;
            }
            *reinterpret_cast<uint4 *>(dst + 8 * g) = pack8(r);
        }
    } else if (EPI == kEpiGatedResidual) {
        __nv_bfloat16 *x = p.out + row * p.n + col;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (8 * g >= nvalid) break;
            float b[8], xv[8], gt[8], r[8];
            unpack8(in.b[g], b);
            unpack8(in.x[g], xv);
            if (p.gate != nullptr) {
                unpack8(in.g[g], gt);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gt[e] = 1.f;
            }
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float2 t = fadd2(make_float2(__uint_as_float(acc[8 * g + e]), __uint_as_float(acc[8 * g + e + 1])),
                                       make_float2(b[e], b[e + 1]));
                const float2 v = ffma2(make_float2(gt[e], gt[e + 1]), t, make_float2(xv[e], xv[e + 1]));
                r[e] = v.x;
                r[e + 1] = v.y;
            }
            *reinterpret_cast<uint4 *>(x + 8 * g) = pack8(r);
        }
    } else {
        __nv_bfloat16 *o = p.out + row * p.n + col;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (8 * g >= nvalid) break;
            float b[8], r[8];
            unpack8(in.b[g], b);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                float2 v = fadd2(make_float2(__uint_as_float(acc[8 * g + e]), __uint_as_float(acc[8 * g + e + 1])),
                                 make_float2(b[e], b[e + 1]));
                if (EPI == kEpiBiasGelu) v = gelu_tanh2(v);
                r[e] = v.x;
                r[e + 1] = v.y;
            }
            if (p.out_packed)
                *reinterpret_cast<uint4 *>(reinterpret_cast<char *>(p.out) + packed_a_offset(row, col + 8 * g, p.n)) =
                    pack8(r);
            else
                *reinterpret_cast<uint4 *>(o + 8 * g) = pack8(r);
        }
    }
}

// PAIR: a cluster of two CTAs works each 256 x 256 tile with cta_group::2
// MMAs issued by its first CTA (rank 0).  Rank r loads A rows [128 r, 128 r +
// 128) and W columns [128 r, 128 r + 128) of the tile into its own shared
// memory, counted on rank 0's stage barrier; each CTA's TMEM holds the fp32
// accumulator of its own 128 rows (all 256 columns), which its own epilogue
// warps drain.  Per SM and K block that is 32 KB of operands for 128 x 256
// x 64 of MMA work, two thirds of what a 128 x 256 tile of one CTA loads.
template <int EPI, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const int S = p.stages;
    const int a_bytes = p.msub * kATileBytes;               // A sub-tiles, then W boxes
    // pair: two K blocks of this CTA's 128 rows of A and 128 columns of W
    const int stage_bytes = PAIR ? 2 * (kATileBytes + 2 * kBBoxBytes) : a_bytes + (p.bn / 64) * kBBoxBytes;
    const int BMt = kBM * p.msub * (PAIR ? 2 : 1);             // rows per tile
    const uint32_t bars = s_base + (uint32_t)(S * stage_bytes);
    // barriers: full[S], empty[S], acc_full[2], acc_empty[2], drain, rope table ready
    auto full = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bars + 8u * (uint32_t)(S + s); };
    auto accf = [&](int b) { return bars + 8u * (uint32_t)(2 * S + b); };
    auto acce = [&](int b) { return bars + 8u * (uint32_t)(2 * S + 2 + b); };
    const uint32_t drain = bars + 8u * (uint32_t)(2 * S + 4);
    const uint32_t rope_ready = bars + 8u * (uint32_t)(2 * S + 5);
    uint8_t *misc = smem + S * stage_bytes + 8 * (2 * S + 6);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 4);
    float2 *rope_tab = reinterpret_cast<float2 *>(misc + 16);   // p.rope_entries of them

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // pair: rank 0 issues the MMAs; both CTAs' loads and epilogue releases
    // count on rank 0's barriers (`lead`)
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    auto lead = [&](uint32_t b) -> uint32_t { return PAIR ? mapa_shared(b, 0) : b; };
    auto wait_lead = [&](uint32_t b, uint32_t parity) -> bool {
        return PAIR ? wait_bar_cluster(b, parity, abort_flag) : wait_bar(b, parity, abort_flag);
    };
    const int cl = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;     // cluster (or CTA)
    const int n_cl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf(b), 1);
            mbar_init(acce(b), PAIR ? 2 * kEpiWarps : kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(rope_ready, kEpiWarps * 32);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        if (PAIR || !p.a_pk) prefetch_tmap(&p.tm_a);
        if (PAIR || !p.w_pk) prefetch_tmap(&p.tm_w);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_holder), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_holder), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();                  // the peer's barriers exist before anything signals them
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int it = 0;                                  // stage loads issued
            bool ok = true;
            for (int t = cl; t < p.n_tiles && ok; t += n_cl) {
                const int m0 = (t / p.n_tiles_n) * BMt, n0 = (t % p.n_tiles_n) * p.bn;
                if (PAIR) {
                    // A stage holds two 64-deep K blocks: [A kb][A kb+1][W kb][W kb+1],
                    // 16 KB each.  Rank r: A rows from m0 + 128 r (loaded if they start
                    // below m) and the W columns from n0 + 128 r that start inside the
                    // matrix; what is not loaded keeps stale data, which reaches only
                    // discarded rows and columns.
                    auto a_in = [&](int r) { return m0 + r * kBM < p.m ? 1 : 0; };
                    auto w_in = [&](int r) {
                        const int c0 = n0 + r * 128;
                        return max(0, min(2, (p.n - c0 + 63) / 64));
                    };
                    const int my_m0 = m0 + (int)rank * kBM, my_n0 = n0 + (int)rank * 128;
                    const int my_a = a_in((int)rank), my_w = w_in((int)rank);
                    for (int kb = 0; kb < p.k_blocks; kb += 2, ++it) {
                        const int nk = min(2, p.k_blocks - kb);
                        const int s = it % S, use = it / S;
                        if (use > 0 && !wait_lead(empty(s), (use - 1) & 1)) {
                            raise_timeout(p, abort_flag);
                            ok = false;
                            break;
                        }
                        const uint32_t sa = s_base + (uint32_t)(s * stage_bytes);
                        const uint32_t fb = lead(full(s));
                        if (rank == 0) {
                            // bytes both CTAs move into this stage: packed A as one 32 KB box
                            // (two adjacent images), packed W as one 16 KB box per K block,
                            // row-major operands as 16 KB A and 8 KB W boxes per K block
                            uint32_t tx = 0;
                            for (int r = 0; r < 2; ++r) {
                                if (a_in(r)) tx += p.a_pk ? 2u * kATileBytes : (uint32_t)(nk * kATileBytes);
                                if (w_in(r) > 0)
                                    tx += (uint32_t)(nk * (p.w_pk ? 2 : w_in(r)) * kBBoxBytes);
                            }
                            mbar_arrive_tx(full(s), tx);
                        }
                        if (my_a) {
                            if (p.a_pk) {
                                // packed A as rows of 256 bytes: the tile's images for K blocks kb
                                // and kb + 1 are adjacent, 64 rows each (with one K block left
                                // the second is the next image or past the end, unused)
                                tma_load_3d_pair(sa, &p.tm_a, fb, 0, ((my_m0 / kBM) * p.kb_total + kb) * 64, 0);
                            } else {
                                for (int j = 0; j < nk; ++j)
                                    tma_load_3d_pair(sa + j * kATileBytes, &p.tm_a, fb, (kb + j) * kBK, my_m0, 0);
                            }
                        }
                        for (int j = 0; j < nk && my_w > 0; ++j) {
                            const uint32_t sw = sa + 2 * kATileBytes + j * 2 * kBBoxBytes;
                            if (p.w_pk) {
                                // this CTA's two 8 KB W images are adjacent: one box of 64 rows of
                                // 256 bytes.  With one image left (n / 64 odd) the box's second
                                // half is the next K block's first image, or past the end (zero
                                // fill): either way it reaches only discarded columns.
                                tma_load_3d_pair(sw, &p.tm_w, fb, 0, ((kb + j) * p.nb_total + my_n0 / 64) * 32, 0);
                            } else {
                                for (int q = 0; q < my_w; ++q)
                                    tma_load_3d_pair(sw + q * kBBoxBytes, &p.tm_w, fb, my_n0 + 64 * q, (kb + j) * kBK, 0);
                            }
                        }
                    }
                    continue;
                }
                // packed B: the tile's 64-column boxes that exist (the rest of
                // the stage keeps stale data, which reaches only discarded columns)
                const int w_boxes = p.w_pk ? min(p.bn / 64, p.nb_total - n0 / 64) : p.bn / 64;
                // A sub-tiles holding rows below m (a sub-tile wholly past m is neither loaded nor multiplied)
                const int a_subs = min(p.msub, (p.m - m0 + kBM - 1) / kBM);
                const uint32_t tx = (uint32_t)(a_subs * kATileBytes + w_boxes * kBBoxBytes);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int s = it % S, use = it / S;
                    if (use > 0 && !wait_bar(empty(s), (use - 1) & 1, abort_flag)) {
                        raise_timeout(p, abort_flag);
                        ok = false;
                        break;
                    }
                    const uint32_t sa = s_base + (uint32_t)(s * stage_bytes);
                    mbar_arrive_tx(full(s), tx);
                    for (int u = 0; u < a_subs; ++u) {
                        if (p.a_pk)
                            bulk_load_1d(sa + u * kATileBytes,
                                         p.a_pk + ((size_t)(m0 / kBM + u) * p.kb_total + kb) * kATileBytes,
                                         kATileBytes, full(s));
                        else
                            tma_load_3d(sa + u * kATileBytes, &p.tm_a, full(s), kb * kBK, m0 + u * kBM, 0);
                    }
                    if (p.w_pk) {
                        bulk_load_1d(sa + a_bytes, p.w_pk + ((size_t)kb * p.nb_total + n0 / 64) * kBBoxBytes,
                                     (uint32_t)(w_boxes * kBBoxBytes), full(s));
                    } else {
                        for (int j = 0; j < p.bn / 64; ++j)
                            tma_load_3d(sa + a_bytes + j * kBBoxBytes, &p.tm_w, full(s), n0 + 64 * j, kb * kBK, 0);
                    }
                }
            }
            // Loads still in flight land before the CTA can exit: wait for
            // the last load of every stage (bounded).  Pair: both CTAs' loads
            // count on rank 0's barriers, and neither CTA leaves before the
            // other (the cluster barrier at the end).
            for (int s = 0; rank == 0 && s < S && s < it; ++s) {
                const int last = ((it - 1 - s) / S) * S + s;   // last load index that used stage s
                mbar_wait(full(s), (last / S) & 1, kWaitNs);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * kBM : kBM, p.bn, 0, 1);
            int it = 0, tc = 0;                          // stages consumed, tiles done
            bool ok = true;
            for (int t = cl; t < p.n_tiles && ok; t += n_cl, ++tc) {
                const int b = tc % p.nbuf, use_b = tc / p.nbuf;
                const int m0 = (t / p.n_tiles_n) * BMt;
                const int a_subs = PAIR ? 1 : min(p.msub, (p.m - m0 + kBM - 1) / kBM);
                if (use_b > 0 && !wait_lead(acce(b), (use_b - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < p.k_blocks; kb += PAIR ? 2 : 1, ++it) {
                    const int s = it % S;
                    if (!wait_lead(full(s), (it / S) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = s_base + (uint32_t)(s * stage_bytes);
                    if (PAIR) {
                        // the stage's K blocks: A at sa + 16 KB j, W at sa + 32 KB + 16 KB j
                        const int nk = min(2, p.k_blocks - kb);
                        for (int j = 0; j < nk; ++j) {
                            const uint64_t da = smem_desc_sw128(sa + j * kATileBytes, 16, 1024);
                            const uint64_t dw = smem_desc_sw128(sa + 2 * kATileBytes + j * 2 * kBBoxBytes, kBBoxBytes, 1024);
                            const uint32_t d_tmem = tmem + (uint32_t)(b * 256);
#pragma unroll
                            for (int kk = 0; kk < kBK / 16; ++kk)
                                mma_ss_pair(d_tmem, da + (uint64_t)((kk * 32) >> 4), dw + (uint64_t)((kk * 2048) >> 4),
                                            idesc, (kb + j > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    const uint64_t dw = smem_desc_sw128(sa + a_bytes, kBBoxBytes, 1024);
                    // sub-tile u accumulates at TMEM column b * 256 + u * bn
                    for (int u = 0; !PAIR && u < a_subs; ++u) {
                        const uint64_t da = smem_desc_sw128(sa + u * kATileBytes, 16, 1024);
                        const uint32_t d_tmem = tmem + (uint32_t)(b * 256 + u * p.bn);
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            mma_ss(d_tmem, da + (uint64_t)((kk * 32) >> 4), dw + (uint64_t)((kk * 2048) >> 4), idesc,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (PAIR) tc_commit_pair(empty(s));
                    else tc_commit(empty(s));
                }
                if (!ok) break;
                if (PAIR) tc_commit_pair(accf(b));
                else tc_commit(accf(b));
            }
            if (!ok) raise_timeout(p, abort_flag);
            // every MMA issued above completes before TMEM is freed
            if (PAIR) tc_commit_pair(drain);
            else tc_commit(drain);
            mbar_wait(drain, 0, kWaitNs);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3, half = (warp - 2) >> 2;
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        int tc = 0;
        bool ok = true;
        const float2 *rope = nullptr;
        if (EPI == kEpiQkvRope && p.rope_entries > 0) {
            // the chunk's rotary angles, once per CTA while the first tile's
            // MMAs run: time pairs per frame, row pairs per row, column
            // pairs per column
            const int nt = p.rope_dt / 2, nd = p.rope_dp / 2;
            const int e_t = p.rope_frames * nt, e_y = p.rope_rows * nd;
            for (int e = threadIdx.x - 64; e < p.rope_entries; e += kEpiWarps * 32) {
                float2 v;
                if (e < e_t) v = rope_angle(e % nt, p.rope_dt, p.t0 + e / nt);
                else if (e < e_t + e_y) v = rope_angle((e - e_t) % nd, p.rope_dp, (e - e_t) / nd);
                else v = rope_angle((e - e_t - e_y) % nd, p.rope_dp, (e - e_t - e_y) / nd);
                rope_tab[e] = v;
            }
            mbar_arrive(rope_ready);
            ok = wait_bar(rope_ready, 0, abort_flag);
            rope = rope_tab;
        }
        // one sub-tile: the two warps of a lane quarter take alternate 32-column
        // chunks; two sub-tiles: warp half u takes all chunks of sub-tile u
        const int sub = p.msub == 2 ? half : 0;
        const int c_first = p.msub == 2 ? 0 : half, c_step = p.msub == 2 ? 1 : 2;
        for (int t = cl; ok && t < p.n_tiles; t += n_cl, ++tc) {
            const int b = tc % p.nbuf, use_b = tc / p.nbuf;
            const int m0 = (t / p.n_tiles_n) * BMt + (int)rank * kBM, n0 = (t % p.n_tiles_n) * p.bn;
            bool w = wait_lead(accf(b), use_b & 1);
            w = __all_sync(0xffffffffu, w);
            if (!w) {
                ok = false;
                break;
            }
            tc_fence_after();
            const long long row = (long long)m0 + sub * kBM + quarter * 32 + lane;
            const bool sub_live = m0 + sub * kBM < p.m;           // warp-uniform
            const bool row_ok = row < p.m;
            int f_pos = 0, y_pos = 0, x_pos = 0;
            if (EPI == kEpiQkvRope) {
                const int f = (int)(row / p.kpf), r = (int)(row - (long long)f * p.kpf);
                f_pos = p.t0 + f;
                y_pos = r / p.grid_w;
                x_pos = r - y_pos * p.grid_w;
            }
            // chunk c's inputs are loaded while chunk c - c_step is computed
            EpiIn in;
            if (sub_live && row_ok && n0 + 32 * c_first < p.n)
                epi_load<EPI>(p, row, n0 + 32 * c_first, min(32, p.n - (n0 + 32 * c_first)), in);
            for (int c = c_first; sub_live && c < p.bn / 32; c += c_step) {
                const int col = n0 + 32 * c;
                if (col >= p.n) break;                   // warp-uniform
                uint32_t acc[32];
                tmem_ld32(tmem + lane_bits + (uint32_t)(b * 256 + sub * p.bn + 32 * c), acc);
                EpiIn next;
                const int col_n = col + 32 * c_step;
                if (row_ok && c + c_step < p.bn / 32 && col_n < p.n)
                    epi_load<EPI>(p, row, col_n, min(32, p.n - col_n), next);
                tmem_wait_ld();
                if (row_ok) epi_chunk<EPI>(p, acc, in, row, col, min(32, p.n - col), f_pos, y_pos, x_pos, rope);
                in = next;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR) mbar_arrive_cluster(lead(acce(b)));
                else mbar_arrive(acce(b));
            }
        }
        if (!ok) raise_timeout(p, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();                  // neither CTA leaves while the pair's MMAs may touch it
    tc_fence_after();
    if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

template <int EPI, bool PAIR>
cudaError_t set_smem_attr_once() {
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        err = cudaFuncSetAttribute(gemm_tc<EPI, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kMaxSmem + 2048 + kRopeTabMax * 8);
    });
    return err;
}

// Tile shape (128 rows by 128, 192 or 256 columns, 256 by 256 on one CTA,
// or 256 by 256 on a CTA pair): the candidate whose rounds of tiles take the
// least time under a model measured on B200.  Per 64-deep K block a tile
// takes the longer of
//   its MMAs: 128 x N x 16 costs 85, 106 or 128 cycles for N = 128, 192,
//     256 (one per k16 step and 128-row sub-tile); the pair's 256 x 256 x 16
//     runs at 128 per SM alone but, with the stage loads in flight, about
//     170 with packed weights and 232 with row-major ones, whose 8 KB boxes
//     take more TMA instructions to issue (measured on the Wan-1.3B
//     projections), and
//   its loads: stages in flight over a loaded round trip of about 4,400
//     cycles (the latency times the bandwidth of the memory system reaching
//     one SM is the shared memory that holds the stages, so a stage's bytes
//     arrive every latency / stages cycles, whatever their size).
// A 256 x 256 tile on one CTA fills TMEM with its two accumulators and
// cannot overlap its epilogue with the next tile's MMAs: it pays about 2,000
// more cycles for a light epilogue (bias, gated residual).  Heavy epilogues
// (GELU's tanh, the rotary sine and cosine) take longer than that per 256 x
// 256 tile (the GELU projection measured 184 against 144 us), so there they
// are not candidates.  A pair's tile holds 128 x 256 per SM, so it keeps two
// accumulator buffers; its rounds are of sms / 2 tiles.
struct TileShape {
    int msub, bn, stages, pair;
};

// A pair's stage holds two K blocks of its 128 rows of A and 128 columns of W.
int stage_bytes_of(int msub, int bn, int pair) {
    return pair ? 2 * (kATileBytes + 2 * kBBoxBytes) : msub * kATileBytes + (bn / 64) * kBBoxBytes;
}

TileShape pick_tile(int m, int n, int k, int sms, int pair_slots, bool heavy_epilogue, bool w_packed) {
    const int k_blocks = (k + kBK - 1) / kBK;
    TileShape best = {1, 256, 4, 0};
    double best_cost = -1.0;
    struct Cand { int msub, bn, pair; };
    for (const Cand c : {Cand{1, 256, 1}, Cand{2, 256, 0}, Cand{1, 256, 0}, Cand{1, 192, 0}, Cand{1, 128, 0}}) {
        if (c.msub == 2 && heavy_epilogue) continue;
        if (c.pair && pair_slots < 1) continue;
        const int stages = std::min(8, kMaxSmem / stage_bytes_of(c.msub, c.bn, c.pair));
        const double mma = c.pair ? 4.0 * (w_packed ? 170.0 : 232.0)
                                  : c.msub * 4.0 * (c.bn == 256 ? 128.0 : c.bn == 192 ? 106.0 : 85.0);
        const double load = 4400.0 / (c.pair ? 2 * stages : stages);   // per K block
        const double epi = !c.pair && c.msub * c.bn > 256 ? 2000.0 : 0.0;
        const int rows = kBM * c.msub * (c.pair ? 2 : 1);
        const long long tiles = (long long)((m + rows - 1) / rows) * ((n + c.bn - 1) / c.bn);
        const int slots = c.pair ? pair_slots : sms;
        const long long rounds = (tiles + slots - 1) / slots;
        const double cost = rounds * (k_blocks * std::max(mma, load) + epi);
        if (best_cost < 0 || cost < best_cost * 0.999) {
            best_cost = cost;
            best = {c.msub, c.bn, stages, c.pair};
        }
    }
    return best;
}

template <int EPI, bool PAIR>
cudaError_t launch_epi(const GemmParams &p, int grid, int smem, cudaStream_t s) {
    const cudaError_t e = set_smem_attr_once<EPI, PAIR>();
    if (e != cudaSuccess) return e;
    cudaError_t le;
    if (PAIR) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        le = cudaLaunchKernelEx(&cfg, gemm_tc<EPI, PAIR>, p);
    } else {
        gemm_tc<EPI, PAIR><<<grid, kThreads, smem, s>>>(p);
        le = cudaGetLastError();
    }
    if (le == cudaSuccess) count_launch();
    return le;
}

// Clusters of two CTAs of gemm_tc<EPI, true> that can be resident at once
// on `device` (at most sms / 2): the two CTAs of a cluster take two SMs of
// one GPC, so a GPC with an odd number of SMs leaves one of them out.  0 if
// the query fails (no pair launches then).
template <int EPI>
int pair_slots_of(int device, int sms) {
    static std::atomic<int> cache[64] = {};
    if (device < 0 || device >= 64) return 0;
    int n = cache[device].load(std::memory_order_relaxed);
    if (n) return n > 0 ? n : 0;
    n = -1;
    if (set_smem_attr_once<EPI, true>() == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (sms / 2 > 0 ? sms / 2 : 1));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kMaxSmem + 2048 + kRopeTabMax * 8;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, gemm_tc<EPI, true>, &cfg) == cudaSuccess && c > 0)
            n = std::min(c, sms / 2);
    }
    cudaGetLastError();
    cache[device].store(n, std::memory_order_relaxed);
    return n > 0 ? n : 0;
}

int pair_slots(int epi, int device, int sms) {
    switch (epi) {
        case kEpiBias: return pair_slots_of<kEpiBias>(device, sms);
        case kEpiBiasGelu: return pair_slots_of<kEpiBiasGelu>(device, sms);
        case kEpiGatedResidual: return pair_slots_of<kEpiGatedResidual>(device, sms);
        default: return pair_slots_of<kEpiQkvRope>(device, sms);
    }
}

template <int EPI>
cudaError_t launch_epi(const GemmParams &p, int grid, int smem, bool pair, cudaStream_t s) {
    return pair ? launch_epi<EPI, true>(p, grid, smem, s) : launch_epi<EPI, false>(p, grid, smem, s);
}

}  // namespace

cudaError_t launch_gemm_bf16(const GemmArgs &g, unsigned *status, int sms, cudaStream_t s) {
    if (g.m <= 0) return cudaSuccess;
    if (g.n < 8 || g.k < 8 || g.n % 8 != 0 || g.k % 8 != 0 || g.epi < 0 || g.epi > kEpiQkvRope)
        return cudaErrorInvalidValue;
    if (g.epi == kEpiQkvRope && (g.n % 3 != 0 || (g.n / 3) % g.head_dim != 0 || g.head_dim % 32 != 0 ||
                                 g.kpf < 1 || g.grid_w < 1))
        return cudaErrorInvalidValue;
    if (!status || sms < 1) return cudaErrorInvalidValue;
    if ((g.a_packed || g.w_packed) && g.k % 64 != 0) return cudaErrorInvalidValue;
    if ((g.w_packed || g.out_packed) && g.n % 64 != 0) return cudaErrorInvalidValue;
    if (g.out_packed && g.epi != kEpiBias && g.epi != kEpiBiasGelu) return cudaErrorInvalidValue;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return cudaErrorInvalidValue;
    // a pair moves packed W two images and packed A two tile images at a time,
    // so it needs at least that many
    const int slots2 = (g.w_packed && packed_b_bytes(g.k, g.n) < 2 * (size_t)kBBoxBytes) ||
                               (g.a_packed && packed_a_bytes(g.m, g.k) < 2 * (size_t)kATileBytes)
                           ? 0
                           : pair_slots(g.epi, device, sms);
    const TileShape ts =
        pick_tile(g.m, g.n, g.k, sms, slots2, g.epi == kEpiBiasGelu || g.epi == kEpiQkvRope, g.w_packed != 0);
    // Row-major operands load by 128-byte-swizzled TMA boxes.  Packed ones
    // load by 1-D bulk copies, or, on a CTA pair (whose loads must count on
    // the first CTA's barrier), by unswizzled boxes of 256-byte rows, which
    // land byte for byte as they lie in memory.
    if (g.a_packed && ts.pair) {
        if (!make_tmap_rows256(&p.tm_a, g.a, packed_a_bytes(g.m, g.k) / 256, 128)) return cudaErrorInvalidValue;
    } else if (!g.a_packed && !make_tmap_bf16(&p.tm_a, g.a, (uint64_t)g.k, (uint64_t)g.m, 1, kBM, 1)) {
        return cudaErrorInvalidValue;
    }
    if (g.w_packed && ts.pair) {
        if (!make_tmap_rows256(&p.tm_w, g.w, packed_b_bytes(g.k, g.n) / 256, 64)) return cudaErrorInvalidValue;
    } else if (!g.w_packed && !make_tmap_bf16(&p.tm_w, g.w, (uint64_t)g.n, (uint64_t)g.k, 1, kBK, 1)) {
        return cudaErrorInvalidValue;
    }
    p.a_pk = g.a_packed ? static_cast<const char *>(g.a) : nullptr;
    p.w_pk = g.w_packed ? static_cast<const char *>(g.w) : nullptr;
    p.kb_total = g.k / 64;
    p.nb_total = g.n / 64;
    p.out_packed = g.out_packed;
    p.m = g.m; p.n = g.n; p.k = g.k;
    p.msub = ts.msub;
    p.bn = ts.bn;
    p.stages = ts.stages;
    p.nbuf = p.msub * p.bn <= 256 ? 2 : 1;
    p.n_tiles_n = (g.n + p.bn - 1) / p.bn;
    const int tile_rows = kBM * p.msub * (ts.pair ? 2 : 1);
    p.n_tiles = ((g.m + tile_rows - 1) / tile_rows) * p.n_tiles_n;
    p.k_blocks = (g.k + kBK - 1) / kBK;
    const int stage_bytes = stage_bytes_of(p.msub, p.bn, ts.pair);
    p.bias = static_cast<const __nv_bfloat16 *>(g.bias);
    p.gate = static_cast<const __nv_bfloat16 *>(g.gate);
    p.out = static_cast<__nv_bfloat16 *>(g.out);
    p.q = static_cast<__nv_bfloat16 *>(g.q);
    p.kk = static_cast<__nv_bfloat16 *>(g.k_out);
    p.v = static_cast<__nv_bfloat16 *>(g.v);
    p.D = g.epi == kEpiQkvRope ? g.n / 3 : g.n;
    p.head_dim = g.head_dim;
    p.kpf = g.kpf;
    p.grid_w = g.grid_w;
    p.t0 = g.t0;
    p.rope_dp = g.head_dim > 0 ? 2 * (g.head_dim / 6) : 0;
    p.rope_dt = g.head_dim - 2 * p.rope_dp;
    if (g.epi == kEpiQkvRope) {
        // rows [0, m) cover frames t0 .. t0 + rope_frames - 1; a frame's rows
        // are rope_rows rows of grid_w columns
        p.rope_frames = (g.m - 1) / g.kpf + 1;
        p.rope_rows = (g.kpf + g.grid_w - 1) / g.grid_w;
        const long long entries = (long long)p.rope_frames * (p.rope_dt / 2) +
                                  (long long)(p.rope_rows + g.grid_w) * (p.rope_dp / 2);
        p.rope_entries = entries <= kRopeTabMax ? (int)entries : 0;
    }
    p.status = status;
    // one CTA (pair: one cluster of two) per SM (pair of SMs) at most
    const int slots = ts.pair ? slots2 : sms;
    const int grid = (p.n_tiles < slots ? p.n_tiles : slots) * (ts.pair ? 2 : 1);
    // stages, barriers (2S + 6), the TMEM holder and the abort flag, the
    // rotary table, plus slack for the 1 KB alignment of the stage ring
    const int smem = p.stages * stage_bytes + 8 * (2 * p.stages + 6) + 16 + p.rope_entries * 8 + 1024;
    const bool pair = ts.pair != 0;
    switch (g.epi) {
        case kEpiBias: return launch_epi<kEpiBias>(p, grid, smem, pair, s);
        case kEpiBiasGelu: return launch_epi<kEpiBiasGelu>(p, grid, smem, pair, s);
        case kEpiGatedResidual: return launch_epi<kEpiGatedResidual>(p, grid, smem, pair, s);
        default: return launch_epi<kEpiQkvRope>(p, grid, smem, pair, s);
    }
}

void gemm_plan_tile(int m, int n, int k, int epi, bool w_packed, int sms, int slots2, int *rows, int *cols,
                    int *pair, int *ctas) {
    const TileShape ts = pick_tile(m, n, k, sms, slots2, epi == kEpiBiasGelu || epi == kEpiQkvRope, w_packed);
    const int tile_rows = kBM * ts.msub * (ts.pair ? 2 : 1);
    const long long tiles = (long long)((m + tile_rows - 1) / tile_rows) * ((n + ts.bn - 1) / ts.bn);
    const int slots = ts.pair ? slots2 : sms;
    *rows = tile_rows;
    *cols = ts.bn;
    *pair = ts.pair;
    *ctas = (int)std::min<long long>(tiles, slots) * (ts.pair ? 2 : 1);
}

void gemm_tile_shape(int m, int n, int k, int epi, int device, int sms, int *rows, int *cols, int *pair,
                     int *ctas) {
    gemm_plan_tile(m, n, k, epi, false, sms, pair_slots(epi, device, sms), rows, cols, pair, ctas);
}

}  // namespace rtr
