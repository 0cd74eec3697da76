// dit_internal.h -- launchers of the DiT-block kernels (dit_block.cu), used by
// the host side of the C ABI (api.cu).  All tensors are row-major, bf16
// unless stated; every launcher returns the CUDA error of its launch.
#pragma once
#include <cuda_runtime.h>

namespace rtr {

// out[i] = LN(x[i]) * (1 + scale) + shift over D channels (eps, no affine);
// scale / shift null: LN(x[i]) alone.  x, out: [n][D]; scale, shift: [D].
cudaError_t launch_ln_modulate(const void *x, const void *shift, const void *scale, void *out, int n, int D,
                               float eps, cudaStream_t s);

// q, k, v ([n][heads][d] = [n][D]) from the fp32 projection qkv ([n][3D]) and
// its bias ([3D]): q and k rotated by the 3D rotary encoding of token i of a
// chunk (frame t0 + i / kpf, row (i % kpf) / grid_w, column i % grid_w).
cudaError_t launch_rope_qkv(const float *qkv, const void *bias, void *q, void *k, void *v, int n, int heads, int d,
                            int kpf, int grid_w, int t0, cudaStream_t s);

// out = in + bias, or GELU(in + bias) (tanh form) when gelu != 0; in fp32
// [n][N], bias and out bf16; N a multiple of 4.
cudaError_t launch_bias_act(const float *in, const void *bias, void *out, int n, int N, int gelu, cudaStream_t s);

// x += gate * (in + bias) in place (gate null: 1); in fp32 [n][D], x bf16.
cudaError_t launch_gated_residual(const float *in, const void *bias, const void *gate, void *x, int n, int D,
                                  cudaStream_t s);

// c = a w with a bf16 [m][k], w bf16 [k][n], c fp32 [m][n], fp32 accumulation
// (cuBLAS GEMM on the given device and stream).
cudaError_t gemm_bf16_f32(int device, cudaStream_t s, const void *a, const void *w, float *c, int m, int n, int k);

}  // namespace rtr
