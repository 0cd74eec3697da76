// kv_copy.cu -- KV-cache update kernel: appends latent frames into the ring
// slots of the reference-preserving rolling cache (papernotes.org note "DiT as
// Real-Time Rerenderer", Method > Key Designs 4), overwrites the anchored
// reference slot, or fills the text cross-attention cache.  Eviction of the
// oldest frame is the overwrite of its slot: no data shifts.
//
// Source rows are [tokens][heads][d] (the layout a QKV projection produces);
// the cache is head-major [heads][rows][d].  The kernel is a pure HBM-bound
// copy: every thread moves four 16-byte vectors, all loads in flight before
// the matching stores, and one grid pass covers K and V together.  Index
// arithmetic uses multiply-high division by run-time constants (Granlund and
// Montgomery, "Division by Invariant Integers using Multiplication", 1994).
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"

namespace rtr {
namespace {

struct FastDiv {
    uint32_t d, m, s;
};

FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    f.s = s;
    // m = floor(2^32 * (2^s - d) / d) + 1; then n / d = (umulhi(n, m) + n) >> s
    // for every n < 2^31.
    f.m = (uint32_t)((((1ull << 32) * ((1ull << s) - d)) / d) + 1);
    return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
    return (__umulhi(n, f.m) + n) >> f.s;
}

struct ScatterDev {
    const uint4 *src[2];
    uint4 *dst[2];
    uint32_t per_tensor;   // 16-byte vectors per tensor (K and V alike)
    uint32_t vpr_log2;     // log2(vectors per (token, head) row)
    FastDiv heads, kfr;
    uint32_t first_slot, slot_mod, slot_off;
    uint64_t rows_per_head;
};

constexpr int kUnroll = 4;
constexpr int kBlock = 256;

// K and V form one index space of 2 * per_tensor vectors; every thread moves
// kUnroll vectors with all its loads in flight before its stores, and the
// grid covers the space in one pass.
__global__ void __launch_bounds__(kBlock) kv_scatter(const ScatterDev a) {
    const uint32_t vmask = (1u << a.vpr_log2) - 1u;
    const uint32_t total = 2u * a.per_tensor;
    const uint32_t base = blockIdx.x * (kBlock * kUnroll) + threadIdx.x;
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const uint32_t i = base + u * kBlock;
        if (i < total) {
            const uint32_t t = i >= a.per_tensor;
            const uint4 *ptr = (t ? a.src[1] : a.src[0]) + (i - t * a.per_tensor);
            asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w)
                         : "l"(ptr));
        }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const uint32_t i = base + u * kBlock;
        if (i < total) {
            const uint32_t t = i >= a.per_tensor;
            const uint32_t j = i - t * a.per_tensor;
            const uint32_t row = j >> a.vpr_log2, c = j & vmask;
            const uint32_t tok = fdiv(row, a.heads);
            const uint32_t h = row - tok * a.heads.d;
            const uint32_t f = fdiv(tok, a.kfr);
            const uint32_t r = tok - f * a.kfr.d;
            uint32_t slot = a.first_slot + f;
            if (slot >= a.slot_mod) slot -= a.slot_mod;
            const uint64_t drow = (uint64_t)(slot + a.slot_off) * a.kfr.d + r;
            (t ? a.dst[1] : a.dst[0])[(((uint64_t)h * a.rows_per_head + drow) << a.vpr_log2) + c] = v[u];
        }
    }
}

}  // namespace

cudaError_t launch_kv_scatter(const ScatterArgs &a, cudaStream_t s) {
    ScatterDev d;
    d.src[0] = static_cast<const uint4 *>(a.src_k);
    d.src[1] = static_cast<const uint4 *>(a.src_v);
    d.dst[0] = static_cast<uint4 *>(a.dst_k);
    d.dst[1] = static_cast<uint4 *>(a.dst_v);
    const uint32_t vpr = (uint32_t)a.row_bytes / 16u;
    uint32_t lg = 0;
    while ((1u << lg) < vpr) ++lg;
    if ((1u << lg) != vpr) return cudaErrorInvalidValue;
    const unsigned long long per_tensor = (unsigned long long)a.n_tok * a.heads * vpr;
    if (per_tensor == 0) return cudaSuccess;
    if (2 * per_tensor >= (1ull << 31)) return cudaErrorInvalidValue;
    d.per_tensor = (uint32_t)per_tensor;
    d.vpr_log2 = lg;
    d.heads = make_fastdiv((uint32_t)a.heads);
    d.kfr = make_fastdiv((uint32_t)a.k_frame);
    d.first_slot = (uint32_t)a.first_slot;
    d.slot_mod = (uint32_t)a.slot_mod;
    d.slot_off = (uint32_t)a.slot_off;
    d.rows_per_head = (uint64_t)a.rows_per_head;
    const unsigned long long per_block = (unsigned long long)kBlock * kUnroll;
    const unsigned long long blocks = (2 * per_tensor + per_block - 1) / per_block;
    kv_scatter<<<(unsigned)blocks, kBlock, 0, s>>>(d);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace rtr
