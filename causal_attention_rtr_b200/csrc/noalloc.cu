// noalloc.cu -- block-causal prefill that allocates no device memory.
//
// rtr_attn_block_causal_prefill keeps its scratch (the partial results of
// attention units split across CTAs) in a buffer the library cudaMallocs on
// first use and grows on demand.  Some callers cannot let a library do that:
// a serving process whose device memory is reserved up front by its own
// caching allocator (an extra cudaMalloc fails or fragments the pool), or a
// frame loop that must not stall, since growing the buffer calls cudaFree,
// which waits for the whole device.  This entry point runs the same kernels
// with the scratch in a file-scope device array instead.
//
// The array is RTR_NOALLOC_SCRATCH_BYTES long and every GPU that loads the
// library holds it until the process exits.  Its device address is looked up
// once per device, on that device's first call.  Every call shares the array
// and it keeps the last call's contents; nothing in it needs to start at zero,
// because every partial result the merge step reads is written earlier in the
// same call.  Calls that overlap on the GPU (on different streams, or from
// different host threads) race on the array and must be ordered by the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "internal.h"
#include "rtr.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[RTR_NOALLOC_SCRATCH_BYTES];

namespace rtr {
namespace {

// Device address of g_noalloc_scratch on `device` (which must be current).
// In host code the array's name only stands in for the symbol; a kernel
// needs the address cudaGetSymbolAddress returns.
void *noalloc_scratch_ptr(int device) {
    static std::mutex mu;
    static void *ptrs[64] = {};
    if (device < 0 || device >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[device]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        ptrs[device] = p;
    }
    return ptrs[device];
}

}  // namespace
}  // namespace rtr

using namespace rtr;

extern "C" rtr_status rtr_attn_block_causal_prefill_noalloc(const void *q, const void *k, const void *v,
                                                            int n_tokens, int heads, int head_dim,
                                                            int k_per_frame, rtr_dtype dt, void *out, float scale,
                                                            int device, rtr_stream_t stream) {
    // The same checks, scale, SM count and schedule as rtr_attn_block_causal_prefill, so
    // that both entry points run identical launches.
    if (n_tokens < 0 || !shape_ok(heads, head_dim) || k_per_frame < 1 || (dt != RTR_BF16 && dt != RTR_F32) ||
        device < 0)
        return RTR_E_INVAL;
    if (n_tokens == 0) return RTR_OK;
    auto aligned16 = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return RTR_E_INVAL;
    if (n_tokens > (1 << 30)) return RTR_E_INVAL;

    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(device) != cudaSuccess) {
        cudaGetLastError();
        return RTR_E_INVAL;
    }
    struct Restore {
        int dev;
        ~Restore() { cudaSetDevice(dev); }
    } restore{prev};

    AttnProblem pb;
    memset(&pb, 0, sizeof(pb));
    pb.nq = n_tokens;
    pb.heads = heads;
    pb.head_dim = head_dim;
    pb.kpf = k_per_frame;
    pb.nseg = 1;
    pb.seg[0] = KvSeg{1, 0, n_tokens, 1};
    pb.scale = resolve_scale(scale, head_dim);
    pb.q = q;
    pb.o = out;
    pb.k1 = k;
    pb.v1 = v;
    pb.rows1 = n_tokens;

    cudaError_t e;
    if (dt == RTR_BF16) {
        AttnPlan plan;
        plan_attn_bf16(pb, sm_count(device), 1, plan);
        // The scratch this launch needs must fit in the static array.
        if (plan.scratch_bytes > (size_t)RTR_NOALLOC_SCRATCH_BYTES) return RTR_E_INVAL;
        void *scratch = noalloc_scratch_ptr(device);
        unsigned *status = device_status_ptr(device);
        if (!scratch || !status) return RTR_E_CUDA;
        e = launch_attn_bf16(pb, plan, nullptr, nullptr, nullptr, status, scratch, (cudaStream_t)stream);
    } else {
        e = launch_attn_f32(pb, (cudaStream_t)stream);   // the fp32 kernel uses no scratch
    }
    if (e == cudaSuccess) return RTR_OK;
    return e == cudaErrorMemoryAllocation ? RTR_E_NOMEM : RTR_E_CUDA;
}
