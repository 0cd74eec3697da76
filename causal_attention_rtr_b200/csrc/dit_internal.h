// dit_internal.h -- launchers of the DiT-block kernels (dit_block.cu), used by
// the host side of the C ABI (api.cu).  All tensors are row-major, bf16
// unless stated; every launcher returns the CUDA error of its launch.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>

namespace rtr {

// Tile-packed operand layouts of the tensor-core projection.  Each holds,
// contiguously, the exact shared-memory image that a 128-byte-swizzled TMA
// box would produce, so one 1-D bulk copy fills a pipeline stage (a tiled
// TMA box moves one 128-byte row per request and reaches about half the
// bulk copy's bytes per clock).
//
// Packed A (activations, K contiguous): element (row, col) of an [m][k]
// matrix, k a multiple of 64, at byte
//     ((row / 128 * (k / 64) + col / 64) * 128 + row % 128) * 128
//     + (((col % 64) / 8) ^ (row % 8)) * 16 + (col % 8) * 2,
// i.e. 16 KB per (128-row tile, 64-column block); ceil(m / 128) row tiles.
// Packed B (weights [k][n], n contiguous): element (kr, nc) at byte
//     ((kr / 64 * (n / 64) + nc / 64) * 64 + kr % 64) * 128
//     + (((nc % 64) / 8) ^ (kr % 8)) * 16 + (nc % 8) * 2,
// 8 KB per (64-row block of k, 64-column block of n); k and n multiples of 64.
__host__ __device__ inline size_t packed_a_offset(long long row, int col, int k) {
    return ((size_t)(row / 128) * (size_t)(k / 64) + (size_t)(col / 64)) * 16384 +
           (size_t)(row % 128) * 128 + (size_t)((((col % 64) / 8) ^ (int)(row % 8)) * 16) + (size_t)(col % 8) * 2;
}
__host__ __device__ inline size_t packed_a_bytes(long long m, int k) {
    return (size_t)((m + 127) / 128) * (size_t)(k / 64) * 16384;
}
__host__ __device__ inline size_t packed_b_bytes(int k, int n) { return (size_t)(k / 64) * (size_t)(n / 64) * 8192; }

// out[i] = LN(x[i]) * (1 + scale) + shift over D channels (eps, no affine);
// scale / shift null: LN(x[i]) alone.  x: [n][D]; scale, shift: [D]; out:
// [n][D], or packed A (D a multiple of 64) when out_packed != 0.
cudaError_t launch_ln_modulate(const void *x, const void *shift, const void *scale, void *out, int n, int D,
                               float eps, cudaStream_t s, int out_packed = 0);

// w [k][n] row-major -> packed B (k, n multiples of 64).
cudaError_t launch_pack_b(const void *w, void *packed, int k, int n, cudaStream_t s);


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
    const void *a;        // bf16 [m][k], 16-byte aligned (packed A when a_packed)
    const void *w;        // bf16 [k][n] ([in][out]), 16-byte aligned (packed B when w_packed)
    int a_packed, w_packed;   // operand in the tile-packed layout (k, and n for B, multiples of 64)
    int out_packed;       // kEpiBias / kEpiBiasGelu: out in packed A layout of [m][n] (n a multiple of 64)
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

// A byte buffer seen as `rows` rows of 256 bytes (128 bf16), boxes of
// box_rows rows, no swizzle: a box lands in shared memory byte for byte as
// it lies in global memory (api.cu).
bool make_tmap_rows256(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows);

// The planner alone, for `sms` SMs of which `pair_slots` CTA pairs can be
// resident at once (0: no pairs), weights packed or row-major.
void gemm_plan_tile(int m, int n, int k, int epi, bool w_packed, int sms, int pair_slots, int *rows, int *cols,
                    int *pair, int *ctas);

// The tile launch_gemm_bf16 picks for an m x n x k product on `device`
// (rows, columns, whether a CTA pair shares it) and the CTAs it launches.
void gemm_tile_shape(int m, int n, int k, int epi, int device, int sms, int *rows, int *cols, int *pair,
                     int *ctas);

}  // namespace rtr
