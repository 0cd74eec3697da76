// attn_f32.cu -- frame-causal attention for float32 storage.
//
// Same problem description (KvSeg runs, frame-causal mask of RTR-DiT's
// 3D attention, papernotes.org note "DiT as Real-Time Rerenderer", Method >
// Key Designs 2) as the tensor-core kernel, computed with fp32 CUDA-core
// arithmetic: one warp per (query row, head), each lane holding D/32 elements
// of the row, a shuffle-reduced dot product per key and an online softmax in
// fp32 with expf.  This is the path of the small fp32 workloads, where exact
// fp32 products matter more than tensor-core throughput.
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"

namespace rtr {
namespace {

template <int D>
__global__ void __launch_bounds__(256) attn_fwd_f32(const AttnProblem p) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const long long warp_id = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const float *Q = static_cast<const float *>(p.q);
    float *O = static_cast<float *>(p.o);
    const long long items = (long long)p.nq * p.heads;
    for (long long item = warp_id; item < items; item += nwarps) {
        const int r = (int)(item / p.heads), h = (int)(item % p.heads);
        float q[E], acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            q[e] = Q[((long long)r * p.heads + h) * D + lane + 32 * e];
            acc[e] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        for (int s = 0; s < p.nseg; ++s) {
            const KvSeg g = p.seg[s];
            int len = g.len;
            if (g.causal) {
                const int lim = (r / p.kpf + 1) * p.kpf;
                len = len < lim ? len : lim;
            }
            const float *Kb = static_cast<const float *>(g.src == 0 ? p.k0 : p.k1);
            const float *Vb = static_cast<const float *>(g.src == 0 ? p.v0 : p.v1);
            for (int j = 0; j < len; ++j) {
                const long long row = (long long)g.row0 + j;
                const long long off = g.src == 0 ? ((long long)h * p.rows0 + row) * D
                                                 : (row * p.heads + h) * D;
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) dot = fmaf(q[e], Kb[off + lane + 32 * e], dot);
#pragma unroll
                for (int w = 16; w > 0; w >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, w);
                const float sc = dot * p.scale;
                const float m_new = fmaxf(m, sc);
                const float corr = expf(m - m_new);
                const float pj = expf(sc - m_new);
                l = l * corr + pj;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] = fmaf(pj, Vb[off + lane + 32 * e], acc[e] * corr);
                m = m_new;
            }
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) O[((long long)r * p.heads + h) * D + lane + 32 * e] = acc[e] * inv;
    }
}

}  // namespace

cudaError_t launch_attn_f32(const AttnProblem &p, cudaStream_t s) {
    const long long items = (long long)p.nq * p.heads;
    long long blocks = (items * 32 + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    if (p.head_dim == 64)
        attn_fwd_f32<64><<<(unsigned)blocks, 256, 0, s>>>(p);
    else if (p.head_dim == 128)
        attn_fwd_f32<128><<<(unsigned)blocks, 256, 0, s>>>(p);
    else
        return cudaErrorInvalidValue;
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace rtr
