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


// Epilogues of the tensor-core projection (gemm_tc.cu), applied to the fp32
// product C = A W before anything is stored; every output is rounded once to
// bf16:
//   kEpiBias           out[m][n] = C + bias
//   kEpiBiasGelu       out[m][n] = GELU_tanh(C + bias)
//   kEpiGatedResidual  out[m][n] += gate * (C + bias) in place (gate null: 1)
//   kEpiQkvRope        n = 3D: q, k, v [m][D] = thirds of C + bias, q and k
//                      turned by the 3D rotary encoding of token i (frame t0 +
//                      i / kpf, row (i % kpf) / grid_w, column i % grid_w) over
//                      heads of head_dim channels
enum { kEpiBias = 0, kEpiBiasGelu = 1, kEpiGatedResidual = 2, kEpiQkvRope = 3 };

struct GemmArgs {
    const void *a;        // bf16 [m][k], 16-byte aligned
    const void *w;        // bf16 [k][n] ([in][out]), 16-byte aligned
    int m, n, k;          // n and k multiples of 8
    int epi;
    const void *bias;     // bf16 [n]
    const void *gate;     // bf16 [n] or null (kEpiGatedResidual)
    void *out;            // bf16 [m][n] (kEpiBias, kEpiBiasGelu, kEpiGatedResidual)
    void *q, *k_out, *v;  // bf16 [m][n / 3] each (kEpiQkvRope)
    int head_dim, kpf, grid_w, t0;   // kEpiQkvRope
};

// C = A W on the tensor cores with the epilogue fused (persistent, up to
// `sms` CTAs); a bounded wait that expires latches RTR_E_TIMEOUT in *status.
cudaError_t launch_gemm_bf16(const GemmArgs &g, unsigned *status, int sms, cudaStream_t s);

}  // namespace rtr
