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
// Structure of one CTA (one head, 256 query rows = two 128-row tiles Q0, Q1):
//   warp 0      TMA producer: Q0/Q1 once, then K_j, V_j into a 4-slot ring
//   warp 1      tcgen05 issuer (one thread): S_i = Q_i K_j^T into TMEM,
//               O_i += P_i V_j with P_i read from TMEM (the "A in tensor
//               memory" form), commits to mbarriers
//   warps 4-7   softmax for Q0, warps 8-11 softmax for Q1: one thread per
//               query row reads its S row from TMEM, online softmax in fp32
//               (exp2 domain, rescale of O only when the running max grows by
//               more than 2^8 -- exact after the final division), writes P
//               as bf16 back over its S columns, and finally normalises O and
//               stores it with TMA.
// The two softmax groups ping-pong: while one works on its S tile the tensor
// core runs the other tile's QK^T or PV.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// Shared memory: Q0, Q1 and 4 K/V slots, each 128 rows x D bf16 stored as D/64
// boxes of 128 rows x 128 bytes with the 128-byte swizzle that TMA writes and
// the tcgen05 descriptors read.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace rtr {

__device__ unsigned g_device_status;   // RTR_OK or RTR_E_TIMEOUT, latched

namespace {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kSlots = 4;         // K/V ring depth
constexpr int kThreads = 384;     // 12 warps
constexpr uint64_t kWaitNs = 1000000000ull;   // bounded waits: 1 s

struct TcParams {
    CUtensorMap tm_q;   // token-major [nq][H][D], box (64, 1, 128)
    CUtensorMap tm_o;   // token-major output
    CUtensorMap tm_k0;  // head-major [H][rows][D], box (64, 128, 1)
    CUtensorMap tm_v0;
    CUtensorMap tm_k1;  // token-major [rows][H][D], box (64, 1, 128)
    CUtensorMap tm_v1;
    int nq, heads, kpf, nseg;
    KvSeg seg[kMaxSegs];
    float scale_log2;   // scale * log2(e)
    unsigned *status;
};

template <int D>
struct Layout {
    static constexpr int kTileBytes = kBM * D * 2;          // one Q / K / V tile
    static constexpr int kQ = 0;                            // Q0, Q1
    static constexpr int kKV = 2 * kTileBytes;              // ring slots
    static constexpr int kBars = kKV + kSlots * kTileBytes; // mbarriers
    // barrier indices
    static constexpr int bQ = 0, bFull = 1, bEmpty = bFull + kSlots, bS = bEmpty + kSlots,
                         bP = bS + 2, bO = bP + 2, bEpi = bO + 2, bDrain = bEpi + 2, kNumBars = bDrain + 1;
    static constexpr int kMisc = kBars + kNumBars * 8;      // tmem holder, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;            // slack for 1 KB alignment
};

__device__ __forceinline__ int seg_len_for(const TcParams &p, int s, int q_last) {
    const KvSeg &g = p.seg[s];
    int len = g.len;
    if (g.causal) {
        const int lim = (q_last / p.kpf + 1) * p.kpf;
        len = len < lim ? len : lim;
    }
    return len;
}

__device__ __forceinline__ void raise_timeout(const TcParams &p, volatile int *abort_flag) {
    *abort_flag = 1;
    atomicExch(p.status, (unsigned)RTR_E_TIMEOUT);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_tc(const __grid_constant__ TcParams p) {
    using L = Layout<D>;
    constexpr int NBOX = D / 64;
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
    const int head = blockIdx.y;
    const int q0 = blockIdx.x * 2 * kBM;
    const int q_last = min(q0 + 2 * kBM - 1, p.nq - 1);

    int T = 0;
    for (int s = 0; s < p.nseg; ++s) T += (seg_len_for(p, s, q_last) + kBN - 1) / kBN;

    if (threadIdx.x == 0) {
        mbar_init(bar(L::bQ), 1);
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(bar(L::bFull + i), 1);
            mbar_init(bar(L::bEmpty + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(L::bS + i), 1);
            mbar_init(bar(L::bP + i), 4);      // one arrive per softmax warp
            mbar_init(bar(L::bO + i), 1);
            mbar_init(bar(L::bEpi + i), kBM);  // every softmax thread
        }
        mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k0);
        prefetch_tmap(&p.tm_v0);
        prefetch_tmap(&p.tm_k1);
        prefetch_tmap(&p.tm_v1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_tx(bar(L::bQ), 2 * L::kTileBytes);
            for (int i = 0; i < 2; ++i)
                for (int b = 0; b < NBOX; ++b)
                    tma_load_3d(sQ + i * L::kTileBytes + b * 16384, &p.tm_q, bar(L::bQ), b * 64, head,
                                q0 + i * kBM);
            int n = 0;
            bool ok = true;
            for (int s = 0; s < p.nseg && ok; ++s) {
                const KvSeg g = p.seg[s];
                const int ntile = (seg_len_for(p, s, q_last) + kBN - 1) / kBN;
                for (int t = 0; t < ntile && ok; ++t) {
                    const int row = g.row0 + t * kBN;
                    for (int kv = 0; kv < 2; ++kv, ++n) {
                        const int slot = n % kSlots, use = n / kSlots;
                        if (use > 0 && !mbar_wait(bar(L::bEmpty + slot), (use - 1) & 1, kWaitNs)) {
                            raise_timeout(p, abort_flag);
                            ok = false;
                            break;
                        }
                        if (*abort_flag) { ok = false; break; }
                        const uint32_t dst = sKV + slot * L::kTileBytes;
                        mbar_arrive_tx(bar(L::bFull + slot), L::kTileBytes);
                        const CUtensorMap *map =
                            g.src == 0 ? (kv ? &p.tm_v0 : &p.tm_k0) : (kv ? &p.tm_v1 : &p.tm_k1);
                        for (int b = 0; b < NBOX; ++b) {
                            if (g.src == 0)
                                tma_load_3d(dst + b * 16384, map, bar(L::bFull + slot), b * 64, row, head);
                            else
                                tma_load_3d(dst + b * 16384, map, bar(L::bFull + slot), b * 64, head, row);
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, 0, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, 0, 1);
            auto issue_s = [&](int i, uint32_t kslot) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
                    const uint64_t a = smem_desc_sw128(sQ + i * L::kTileBytes + off, 16, 1024);
                    const uint64_t b = smem_desc_sw128(kslot + off, 16, 1024);
                    mma_ss(tmem + i * 128, a, b, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](int i, uint32_t vslot, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint64_t b = smem_desc_sw128(vslot + kk * 2048, 16384, 1024);
                    mma_ts(tmem + 256 + i * D, tmem + i * 128 + kk * 8, b, idesc_o, (acc || kk > 0) ? 1u : 0u);
                }
            };
            int n = 0;
            bool ok = mbar_wait(bar(L::bQ), 0, kWaitNs);
            uint32_t kslot = 0;
            if (ok) {
                const int slot = n % kSlots;
                ok = mbar_wait(bar(L::bFull + slot), (n / kSlots) & 1, kWaitNs);
                if (ok) {
                    tc_fence_after();
                    kslot = sKV + slot * L::kTileBytes;
                    issue_s(0, kslot);
                    tc_commit(bar(L::bS + 0));
                    issue_s(1, kslot);
                    tc_commit(bar(L::bS + 1));
                    tc_commit(bar(L::bEmpty + slot));
                    ++n;
                }
            }
            for (int j = 0; j < T && ok; ++j) {
                const int vs = n % kSlots;
                ok = mbar_wait(bar(L::bFull + vs), (n / kSlots) & 1, kWaitNs);
                if (!ok) break;
                ++n;
                const uint32_t vslot = sKV + vs * L::kTileBytes;
                ok = mbar_wait(bar(L::bP + 0), j & 1, kWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                issue_pv(0, vslot, j > 0);
                if (j == T - 1) tc_commit(bar(L::bO + 0));
                int ks = -1;
                if (j + 1 < T) {
                    ks = n % kSlots;
                    ok = mbar_wait(bar(L::bFull + ks), (n / kSlots) & 1, kWaitNs);
                    if (!ok) break;
                    tc_fence_after();
                    kslot = sKV + ks * L::kTileBytes;
                    issue_s(0, kslot);
                    tc_commit(bar(L::bS + 0));
                }
                ok = mbar_wait(bar(L::bP + 1), j & 1, kWaitNs) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                issue_pv(1, vslot, j > 0);
                tc_commit(bar(L::bEmpty + vs));
                if (j == T - 1) tc_commit(bar(L::bO + 1));
                if (j + 1 < T) {
                    issue_s(1, kslot);
                    tc_commit(bar(L::bS + 1));
                    tc_commit(bar(L::bEmpty + ks));
                    ++n;
                }
            }
            if (!ok) raise_timeout(p, abort_flag);
            // Drain: every MMA issued above has completed before TMEM is freed.
            tc_commit(bar(L::bDrain));
            mbar_wait(bar(L::bDrain), 0, kWaitNs);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax
        const int i = (warp - 4) >> 2;                  // which query tile
        const int sub = warp & 3;                       // TMEM lane quarter
        const int row_local = sub * 32 + lane;
        const int q_row = q0 + i * kBM + row_local;
        const int row_vis_end = (q_row / p.kpf + 1) * p.kpf;
        const uint32_t lane_bits = (uint32_t)(sub * 32) << 16;
        const uint32_t tS = tmem + lane_bits + i * 128;
        const uint32_t tO = tmem + lane_bits + 256 + i * D;
        const float sl2 = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int j = 0;
        for (int s = 0; s < p.nseg && ok; ++s) {
            const KvSeg g = p.seg[s];
            const int ntile = (seg_len_for(p, s, q_last) + kBN - 1) / kBN;
            const int row_len = g.causal ? min(g.len, row_vis_end) : g.len;
            for (int t = 0; t < ntile; ++t, ++j) {
                const int lim = row_len - t * kBN;      // visible columns of this row
                bool w = !*abort_flag && mbar_wait(bar(L::bS + i), j & 1, kWaitNs);
                w = __all_sync(0xffffffffu, w);
                if (!w) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[128];
                tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                tmem_wait_ld();
                float *sv = reinterpret_cast<float *>(sr);
                if (lim < kBN) {
#pragma unroll
                    for (int c = 0; c < kBN; ++c)
                        if (c >= lim) sv[c] = -INFINITY;
                }
                float mx = sv[0];
#pragma unroll
                for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, sv[c]);
                const float m_new = fmaxf(m_run, mx * sl2);
                const bool upd = m_new > m_run + 8.0f;
                float factor = 1.f;
                if (upd) {
                    factor = fast_exp2(m_run - m_new);
                    m_run = m_new;
                    l_run *= factor;
                }
                if (j > 0 && __any_sync(0xffffffffu, upd)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                        tmem_st32(tO + 32 * c, o);
                    }
                }
                const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float p0 = fast_exp2(fmaf(sv[64 * h + 2 * e], sl2, neg_m));
                        const float p1 = fast_exp2(fmaf(sv[64 * h + 2 * e + 1], sl2, neg_m));
                        sum += p0 + p1;
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tS + 32 * h, pk);
                }
                l_run += sum;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::bP + i));
            }
        }
        // ------------------------------------------------------------ epilogue
        const uint32_t sOut = sQ + i * L::kTileBytes;   // Q_i is dead once O_i is final
        bool w = ok && !*abort_flag && mbar_wait(bar(L::bO + i), 0, kWaitNs);
        w = __all_sync(0xffffffffu, w);
        if (w) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(o[8 * t + 0]) * inv, __uint_as_float(o[8 * t + 1]) * inv);
                    v.y = pack_bf16x2(__uint_as_float(o[8 * t + 2]) * inv, __uint_as_float(o[8 * t + 3]) * inv);
                    v.z = pack_bf16x2(__uint_as_float(o[8 * t + 4]) * inv, __uint_as_float(o[8 * t + 5]) * inv);
                    v.w = pack_bf16x2(__uint_as_float(o[8 * t + 6]) * inv, __uint_as_float(o[8 * t + 7]) * inv);
                    const int col = 32 * c + 8 * t;
                    const int box = col / 64, cc = (col % 64) / 8;
                    const uint32_t addr = sOut + box * 16384 + row_local * 128 + ((cc ^ (row_local & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                                 "r"(v.z), "r"(v.w)
                                 : "memory");
                }
            }
            fence_proxy_async_smem();
        } else if (ok) {
            raise_timeout(p, abort_flag);
        }
        mbar_arrive(bar(L::bEpi + i));
        if (row_local == 0) {
            const bool all = mbar_wait(bar(L::bEpi + i), 0, kWaitNs);
            if (all && w && !*abort_flag && q0 + i * kBM < p.nq) {
                for (int b = 0; b < NBOX; ++b) tma_store_3d(&p.tm_o, sOut + b * 16384, b * 64, head, q0 + i * kBM);
                bulk_commit();
                bulk_wait_read0();
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
cudaError_t launch_tc(const TcParams &tp, int nq, int heads, cudaStream_t s) {
    using L = Layout<D>;
    static int configured_mask = 0;   // per device bit (up to 32 devices)
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(configured_mask & (1 << dev))) {
        cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return e;
        configured_mask |= 1 << dev;
    }
    dim3 grid((nq + 2 * kBM - 1) / (2 * kBM), heads);
    attn_fwd_tc<D><<<grid, kThreads, L::kAlloc, s>>>(tp);
    return cudaGetLastError();
}

}  // namespace

unsigned *device_status_ptr(int device) {
    static unsigned *ptrs[64] = {};
    if (device < 0 || device >= 64) return nullptr;
    if (!ptrs[device]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        ptrs[device] = static_cast<unsigned *>(p);
    }
    return ptrs[device];
}

cudaError_t launch_attn_bf16(const AttnProblem &p, const CUtensorMap *tm_k0, const CUtensorMap *tm_v0,
                             unsigned *status, cudaStream_t s) {
    TcParams tp;
    memset(&tp, 0, sizeof(tp));
    const uint64_t D = (uint64_t)p.head_dim;
    if (!make_tmap_bf16(&tp.tm_q, p.q, D, p.heads, p.nq, 1, kBM)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&tp.tm_o, p.o, D, p.heads, p.nq, 1, kBM)) return cudaErrorInvalidValue;
    bool have0 = false, have1 = false;
    for (int i = 0; i < p.nseg; ++i) (p.seg[i].src == 0 ? have0 : have1) = true;
    if (have1) {
        if (!make_tmap_bf16(&tp.tm_k1, p.k1, D, p.heads, p.rows1, 1, kBN)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16(&tp.tm_v1, p.v1, D, p.heads, p.rows1, 1, kBN)) return cudaErrorInvalidValue;
    } else {
        tp.tm_k1 = tp.tm_q;   // never read; any valid map
        tp.tm_v1 = tp.tm_q;
    }
    if (have0) {
        tp.tm_k0 = *tm_k0;
        tp.tm_v0 = *tm_v0;
    } else {
        tp.tm_k0 = tp.tm_q;
        tp.tm_v0 = tp.tm_q;
    }
    tp.nq = p.nq;
    tp.heads = p.heads;
    tp.kpf = p.kpf;
    tp.nseg = p.nseg;
    for (int i = 0; i < p.nseg; ++i) tp.seg[i] = p.seg[i];
    tp.scale_log2 = p.scale * 1.4426950408889634f;
    tp.status = status;
    if (p.head_dim == 128) return launch_tc<128>(tp, p.nq, p.heads, s);
    if (p.head_dim == 64) return launch_tc<64>(tp, p.nq, p.heads, s);
    return cudaErrorInvalidValue;
}

}  // namespace rtr
