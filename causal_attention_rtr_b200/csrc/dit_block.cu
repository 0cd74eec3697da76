// dit_block.cu -- the layer norms of one DiT block around the frame-causal
// attention (the projections and their bias / rotary / GELU / gated-residual
// epilogues are the tensor-core GEMM of gemm_tc.cu).
//
// Sources: papernotes.org note "DiT as Real-Time Rerenderer", Method >
// Overall Architecture (DiT blocks over the patchified tokens, conditioned on
// the diffusion timestep) and Key Designs 1 (text through cross attention).
// The block's internals are readings of those pages: layer norms without
// affine (eps 1e-6) modulated by per-channel shift / scale vectors; the
// normalised row is rounded once to bf16 (round to nearest even).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dit_internal.h"
#include "internal.h"

namespace rtr {
namespace {

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

// Sum over the block (blockDim.x a multiple of 32, at most 1024).
__device__ float block_sum(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();                        // red[] free from a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    return t;
}

// One block per row: mean, then variance around it, then the normalised and
// modulated row; the row (a few KB) is re-read from L1/L2 in each pass.
__global__ void __launch_bounds__(256) ln_modulate(const __nv_bfloat16 *x, const __nv_bfloat16 *shift,
                                                   const __nv_bfloat16 *scale, __nv_bfloat16 *out, int D,
                                                   float eps) {
    __shared__ float red[32];
    const size_t row = blockIdx.x;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * D);
    const int nv = D / 8;
    float s = 0.f;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        float f[8];
        unpack8(xr[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) s += f[e];
    }
    const float mean = block_sum(s, red) / (float)D;
    float q = 0.f;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        float f[8];
        unpack8(xr[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) q += (f[e] - mean) * (f[e] - mean);
    }
    const float rstd = 1.0f / sqrtf(block_sum(q, red) / (float)D + eps);
    uint4 *orow = reinterpret_cast<uint4 *>(out + row * D);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        float f[8];
        unpack8(xr[i], f);
        if (scale != nullptr) {
            float sc[8], sh[8];
            unpack8(reinterpret_cast<const uint4 *>(scale)[i], sc);
            unpack8(reinterpret_cast<const uint4 *>(shift)[i], sh);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (f[e] - mean) * rstd * (1.0f + sc[e]) + sh[e];
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (f[e] - mean) * rstd;
        }
        orow[i] = make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
    }
}

// One CTA per row with one 8-channel vector per thread held in registers
// (D <= 8192): the row is read once; mean and variance around it by two block
// sums; the normalised, modulated row in one rounding.
__global__ void __launch_bounds__(1024) ln_modulate_reg(const __nv_bfloat16 *x, const __nv_bfloat16 *shift,
                                                        const __nv_bfloat16 *scale, __nv_bfloat16 *out, int D,
                                                        float eps, int out_packed) {
    __shared__ float red[32];
    const size_t row = blockIdx.x;
    const int nv = D / 8, i = threadIdx.x;
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (i < nv) unpack8(reinterpret_cast<const uint4 *>(x + row * D)[i], f);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) s += f[e];
    const float mean = block_sum(s, red) / (float)D;
    float q = 0.f;
    if (i < nv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) q += (f[e] - mean) * (f[e] - mean);
    }
    const float rstd = 1.0f / sqrtf(block_sum(q, red) / (float)D + eps);
    if (i >= nv) return;
    if (scale != nullptr) {
        float sc[8], sh[8];
        unpack8(reinterpret_cast<const uint4 *>(scale)[i], sc);
        unpack8(reinterpret_cast<const uint4 *>(shift)[i], sh);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = (f[e] - mean) * rstd * (1.0f + sc[e]) + sh[e];
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = (f[e] - mean) * rstd;
    }
    const uint4 v = make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
    if (out_packed)
        *reinterpret_cast<uint4 *>(reinterpret_cast<char *>(out) + packed_a_offset((long long)row, 8 * i, D)) = v;
    else
        reinterpret_cast<uint4 *>(out + row * D)[i] = v;
}

// One warp per row, the row in registers (VPL 8-channel vectors a lane, D <=
// 256 VPL): mean and variance by warp shuffles, no shared memory and no
// block barrier, eight rows a CTA, so every row of a chunk is in flight at
// once (the one-CTA-per-row kernel above ran about three waves of small CTAs
// with two block barriers each).  Same arithmetic as ln_modulate_reg; only
// the order of the fp32 sums differs.
template <int VPL>
__global__ void __launch_bounds__(256) ln_modulate_warp(const __nv_bfloat16 *x, const __nv_bfloat16 *shift,
                                                       const __nv_bfloat16 *scale, __nv_bfloat16 *out, int n, int D,
                                                       float eps, int out_packed) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= n) return;
    const int nv = D / 8;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * D);
    float f[VPL][8];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int i = lane + 32 * j;
        if (i < nv) {
            unpack8(xr[i], f[j]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[j][e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) s += f[j][e];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)D;
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        if (lane + 32 * j < nv) {
#pragma unroll
            for (int e = 0; e < 8; ++e) q += (f[j][e] - mean) * (f[j][e] - mean);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = 1.0f / sqrtf(q / (float)D + eps);
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int i = lane + 32 * j;
        if (i >= nv) break;
        if (scale != nullptr) {
            float sc[8], sh[8];
            unpack8(reinterpret_cast<const uint4 *>(scale)[i], sc);
            unpack8(reinterpret_cast<const uint4 *>(shift)[i], sh);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[j][e] = (f[j][e] - mean) * rstd * (1.0f + sc[e]) + sh[e];
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[j][e] = (f[j][e] - mean) * rstd;
        }
        const uint4 v = make_uint4(pack2(f[j][0], f[j][1]), pack2(f[j][2], f[j][3]), pack2(f[j][4], f[j][5]),
                                   pack2(f[j][6], f[j][7]));
        if (out_packed)
            *reinterpret_cast<uint4 *>(reinterpret_cast<char *>(out) + packed_a_offset(row, 8 * i, D)) = v;
        else
            reinterpret_cast<uint4 *>(out + row * D)[i] = v;
    }
}

// One thread per 16-byte piece of w: its 8 n-consecutive elements move to
// their place in the packed layout.
__global__ void __launch_bounds__(256) pack_b(const uint4 *w, char *out, int k, int n8) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)k * n8) return;
    const int kr = (int)(idx / n8), c8 = (int)(idx - (long long)kr * n8);
    const int n = n8 * 8, nc = c8 * 8;
    const size_t off = ((size_t)(kr / 64) * (size_t)(n / 64) + (size_t)(nc / 64)) * 8192 + (size_t)(kr % 64) * 128 +
                       (size_t)((((nc % 64) / 8) ^ (kr % 8)) * 16);
    *reinterpret_cast<uint4 *>(out + off) = w[idx];
}

cudaError_t launched() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

cudaError_t launch_ln_modulate(const void *x, const void *shift, const void *scale, void *out, int n, int D,
                               float eps, cudaStream_t s, int out_packed) {
    if (n <= 0) return cudaSuccess;
    if (D % 8 != 0 || (scale == nullptr) != (shift == nullptr)) return cudaErrorInvalidValue;
    if (out_packed && (D % 64 != 0 || D / 8 > 1024)) return cudaErrorInvalidValue;
    const int vpl = (D / 8 + 31) / 32;          // 8-channel vectors a lane, one warp per row
    if (vpl <= 8) {
        const auto *xx = static_cast<const __nv_bfloat16 *>(x);
        const auto *sh = static_cast<const __nv_bfloat16 *>(shift);
        const auto *sc = static_cast<const __nv_bfloat16 *>(scale);
        auto *o = static_cast<__nv_bfloat16 *>(out);
        const unsigned grid = (unsigned)((n + 7) / 8);
        switch (vpl) {
            case 1: ln_modulate_warp<1><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            case 2: ln_modulate_warp<2><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            case 3: ln_modulate_warp<3><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            case 4: ln_modulate_warp<4><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            case 5: ln_modulate_warp<5><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            case 6: ln_modulate_warp<6><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            case 7: ln_modulate_warp<7><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
            default: ln_modulate_warp<8><<<grid, 256, 0, s>>>(xx, sh, sc, o, n, D, eps, out_packed); break;
        }
        return launched();
    }
    if (D / 8 <= 1024) {
        const int threads = (D / 8 + 31) / 32 * 32;
        ln_modulate_reg<<<n, threads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(shift),
            static_cast<const __nv_bfloat16 *>(scale), static_cast<__nv_bfloat16 *>(out), D, eps, out_packed);
        return launched();
    }
    ln_modulate<<<n, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(shift),
                                  static_cast<const __nv_bfloat16 *>(scale), static_cast<__nv_bfloat16 *>(out), D,
                                  eps);
    return launched();
}

cudaError_t launch_pack_b(const void *w, void *packed, int k, int n, cudaStream_t s) {
    if (k <= 0 || n <= 0) return cudaSuccess;
    if (k % 64 != 0 || n % 64 != 0) return cudaErrorInvalidValue;
    const long long total = (long long)k * (n / 8);
    pack_b<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(static_cast<const uint4 *>(w), static_cast<char *>(packed), k,
                                                            n / 8);
    return launched();
}

}  // namespace rtr
