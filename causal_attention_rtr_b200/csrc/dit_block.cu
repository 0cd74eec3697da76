// dit_block.cu -- the kernels of one DiT block around the frame-causal
// attention: modulated layer norm, the 3D rotary encoding of the queries and
// keys, bias / tanh-GELU and gated-residual epilogues of the projections, and
// the projections themselves (cuBLAS GEMMs with fp32 outputs).
//
// Sources: papernotes.org note "DiT as Real-Time Rerenderer", Method >
// Overall Architecture (DiT blocks over the patchified tokens, conditioned on
// the diffusion timestep) and Key Designs 1 (text through cross attention);
// gist.science explainer "Adapting VACE for Real-Time Autoregressive Video
// Diffusion", section 1 (rotary encodings baked into cached keys).  The
// block's internals are readings of those pages: layer norms without affine
// (eps 1e-6) modulated by per-channel shift / scale / gate vectors, the
// rotary form of Su et al., "RoFormer" (2021), eq. 13-15, split over
// (frame, row, column) parts of d - 2P, P, P channels with P = 2 floor(d/6),
// and the tanh form of GELU.  Every tensor the next step consumes is
// rounded once to bf16 (round to nearest even); the rest is fp32.
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "dit_internal.h"
#include "internal.h"

namespace rtr {
namespace {

constexpr float kLog2RopeBase = 13.287712379549449f;   // log2(10000)

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
                                                        float eps) {
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
    reinterpret_cast<uint4 *>(out + row * D)[i] =
        make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

// One thread per (token, head, channel pair): bias, rotation of the q and k
// pairs by the pair's angle, v copied; outputs rounded once to bf16.
__global__ void __launch_bounds__(256) rope_qkv(const float *qkv, const __nv_bfloat16 *bias, __nv_bfloat16 *q,
                                                __nv_bfloat16 *k, __nv_bfloat16 *v, long long total, int heads,
                                                int d, int kpf, int grid_w, int t0, int dt, int dp) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int half = d / 2;
    const int pr = (int)(idx % half);
    const long long rest = idx / half;
    const int h = (int)(rest % heads);
    const long long i = rest / heads;
    const int D = heads * d;
    const int c = 2 * pr, col = h * d + c;
    const float *row = qkv + i * 3 * (long long)D;
    const float2 bq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(bias + col));
    const float2 bk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(bias + D + col));
    const float2 bv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(bias + 2 * D + col));
    const float q0 = row[col] + bq.x, q1 = row[col + 1] + bq.y;
    const float k0 = row[D + col] + bk.x, k1 = row[D + col + 1] + bk.y;
    const float v0 = row[2 * D + col] + bv.x, v1 = row[2 * D + col + 1] + bv.y;
    const int f = (int)(i / kpf), r = (int)(i - (long long)f * kpf);
    const int y = r / grid_w, xcol = r - y * grid_w;
    int j, size, pos;
    if (c < dt) {
        j = pr; size = dt; pos = t0 + f;
    } else if (c < dt + dp) {
        j = (c - dt) / 2; size = dp; pos = y;
    } else {
        j = (c - dt - dp) / 2; size = dp; pos = xcol;
    }
    const float theta = exp2f(-(float)(2 * j) / (float)size * kLog2RopeBase);
    float sn, cs;
    sincosf((float)pos * theta, &sn, &cs);
    const long long o = i * D + col;
    *reinterpret_cast<uint32_t *>(q + o) = pack2(q0 * cs - q1 * sn, q0 * sn + q1 * cs);
    *reinterpret_cast<uint32_t *>(k + o) = pack2(k0 * cs - k1 * sn, k0 * sn + k1 * cs);
    *reinterpret_cast<uint32_t *>(v + o) = pack2(v0, v1);
}

__device__ __forceinline__ float gelu_tanh(float x) {
    const float kS = 0.7978845608028654f;   // sqrt(2 / pi)
    return 0.5f * x * (1.0f + tanhf(kS * (x + 0.044715f * x * x * x)));
}

// Four consecutive elements per thread.
__global__ void __launch_bounds__(256) bias_act(const float4 *in, const __nv_bfloat16 *bias, uint2 *out,
                                                long long total4, int N4, int gelu) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total4) return;
    const int c4 = (int)(idx % N4);
    const float4 a = in[idx];
    const uint2 bb = reinterpret_cast<const uint2 *>(bias)[c4];
    float f[4] = {a.x + __uint_as_float(bb.x << 16), a.y + __uint_as_float(bb.x & 0xffff0000u),
                  a.z + __uint_as_float(bb.y << 16), a.w + __uint_as_float(bb.y & 0xffff0000u)};
    if (gelu) {
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] = gelu_tanh(f[e]);
    }
    out[idx] = make_uint2(pack2(f[0], f[1]), pack2(f[2], f[3]));
}

__global__ void __launch_bounds__(256) gated_residual(const float4 *in, const __nv_bfloat16 *bias,
                                                      const __nv_bfloat16 *gate, uint2 *x, long long total4,
                                                      int D4) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total4) return;
    const int c4 = (int)(idx % D4);
    const float4 a = in[idx];
    const uint2 bb = reinterpret_cast<const uint2 *>(bias)[c4];
    const uint2 xx = x[idx];
    float g[4] = {1.f, 1.f, 1.f, 1.f};
    if (gate != nullptr) {
        const uint2 gg = reinterpret_cast<const uint2 *>(gate)[c4];
        g[0] = __uint_as_float(gg.x << 16); g[1] = __uint_as_float(gg.x & 0xffff0000u);
        g[2] = __uint_as_float(gg.y << 16); g[3] = __uint_as_float(gg.y & 0xffff0000u);
    }
    const float r0 = __uint_as_float(xx.x << 16) + g[0] * (a.x + __uint_as_float(bb.x << 16));
    const float r1 = __uint_as_float(xx.x & 0xffff0000u) + g[1] * (a.y + __uint_as_float(bb.x & 0xffff0000u));
    const float r2 = __uint_as_float(xx.y << 16) + g[2] * (a.z + __uint_as_float(bb.y << 16));
    const float r3 = __uint_as_float(xx.y & 0xffff0000u) + g[3] * (a.w + __uint_as_float(bb.y & 0xffff0000u));
    x[idx] = make_uint2(pack2(r0, r1), pack2(r2, r3));
}

unsigned blocks_for(long long n, int threads) { return (unsigned)((n + threads - 1) / threads); }

cudaError_t launched() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

cudaError_t launch_ln_modulate(const void *x, const void *shift, const void *scale, void *out, int n, int D,
                               float eps, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    if (D % 8 != 0 || (scale == nullptr) != (shift == nullptr)) return cudaErrorInvalidValue;
    if (D / 8 <= 1024) {
        const int threads = (D / 8 + 31) / 32 * 32;
        ln_modulate_reg<<<n, threads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(shift),
            static_cast<const __nv_bfloat16 *>(scale), static_cast<__nv_bfloat16 *>(out), D, eps);
        return launched();
    }
    ln_modulate<<<n, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(shift),
                                  static_cast<const __nv_bfloat16 *>(scale), static_cast<__nv_bfloat16 *>(out), D,
                                  eps);
    return launched();
}

cudaError_t launch_rope_qkv(const float *qkv, const void *bias, void *q, void *k, void *v, int n, int heads, int d,
                            int kpf, int grid_w, int t0, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int dp = 2 * (d / 6), dt = d - 2 * dp;
    const long long total = (long long)n * heads * (d / 2);
    rope_qkv<<<blocks_for(total, 256), 256, 0, s>>>(qkv, static_cast<const __nv_bfloat16 *>(bias),
                                                    static_cast<__nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(k),
                                                    static_cast<__nv_bfloat16 *>(v), total, heads, d, kpf, grid_w,
                                                    t0, dt, dp);
    return launched();
}

cudaError_t launch_bias_act(const float *in, const void *bias, void *out, int n, int N, int gelu, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    if (N % 4 != 0) return cudaErrorInvalidValue;
    const long long total4 = (long long)n * (N / 4);
    bias_act<<<blocks_for(total4, 256), 256, 0, s>>>(reinterpret_cast<const float4 *>(in),
                                                     static_cast<const __nv_bfloat16 *>(bias),
                                                     static_cast<uint2 *>(out), total4, N / 4, gelu);
    return launched();
}

cudaError_t launch_gated_residual(const float *in, const void *bias, const void *gate, void *x, int n, int D,
                                  cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    if (D % 4 != 0) return cudaErrorInvalidValue;
    const long long total4 = (long long)n * (D / 4);
    gated_residual<<<blocks_for(total4, 256), 256, 0, s>>>(
        reinterpret_cast<const float4 *>(in), static_cast<const __nv_bfloat16 *>(bias),
        static_cast<const __nv_bfloat16 *>(gate), static_cast<uint2 *>(x), total4, D / 4);
    return launched();
}

// One cuBLAS handle per (device, stream), created on first use and kept.
cudaError_t gemm_bf16_f32(int device, cudaStream_t s, const void *a, const void *w, float *c, int m, int n, int k) {
    static std::mutex mu;
    static std::map<std::pair<int, cudaStream_t>, cublasHandle_t> handles;
    cublasHandle_t h = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = handles.find({device, s});
        if (it == handles.end()) {
            if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return cudaErrorUnknown;
            if (cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS) {
                cublasDestroy(h);
                return cudaErrorUnknown;
            }
            handles[{device, s}] = h;
        } else {
            h = it->second;
        }
    }
    // Row-major c[m][n] = a[m][k] w[k][n] is column-major c^T = w^T a^T.
    const float alpha = 1.f, beta = 0.f;
    const cublasStatus_t st = cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, n, m, k, &alpha, w, CUDA_R_16BF, n, a,
                                           CUDA_R_16BF, k, &beta, c, CUDA_R_32F, n, CUBLAS_COMPUTE_32F,
                                           CUBLAS_GEMM_DEFAULT);
    return st == CUBLAS_STATUS_SUCCESS ? cudaGetLastError() : cudaErrorUnknown;
}

}  // namespace rtr
