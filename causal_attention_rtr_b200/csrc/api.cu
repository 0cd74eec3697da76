// api.cu -- host side of librtr: the C ABI declared in include/rtr.h.
//
// Owns the KV-cache and cross-attention buffers, keeps the host-side index
// maps of the reference-preserving rolling cache (papernotes.org note "DiT as
// Real-Time Rerenderer", Method > Key Designs 4), validates every argument
// before anything is enqueued, turns the cache state into the list of key runs
// the attention kernels read, and launches the kernels.  No compute happens
// here and there is no host fallback: every data operation is a kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <map>
#include <mutex>
#include <cstdint>
#include <cstring>
#include <new>
#include <tuple>
#include <utility>
#include <vector>

#include "dit_internal.h"
#include "internal.h"
#include "rtr.h"

namespace rtr {

// ------------------------------------------------------------------ tensor maps
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_fn() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
}

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = lookup_encode_fn();   // initialised once, thread-safe
    return fn;
}

struct DeviceGuard {
    int prev = -1;
    bool ok = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) return;
        ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elt_size(rtr_dtype dt) { return dt == RTR_BF16 ? 2 : 4; }

}  // namespace

bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t d, uint64_t mid, uint64_t outer,
                    uint32_t box_mid, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || !aligned16(base)) return false;
    cuuint64_t dims[3] = {d, mid, outer};
    cuuint64_t strides[2] = {d * 2, mid * d * 2};
    cuuint32_t box[3] = {64, box_mid, box_outer};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_strided(CUtensorMap *m, const void *base, uint64_t d, uint64_t mid, uint64_t outer,
                            uint64_t stride_outer, uint32_t box_mid, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || !aligned16(base)) return false;
    cuuint64_t dims[3] = {d, mid, outer};
    cuuint64_t strides[2] = {d * 2, stride_outer};
    cuuint32_t box[3] = {64, box_mid, box_outer};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_rows256(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || !aligned16(base) || rows < box_rows) return false;
    cuuint64_t dims[3] = {128, rows, 1};
    cuuint64_t strides[2] = {256, rows * 256};
    cuuint32_t box[3] = {128, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {
std::atomic<unsigned long long> g_launches{0};
}

void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// Device allocations of the library go through lib_malloc, so that a test can
// make chosen ones fail (rtr_test_fail_allocs) and check the RTR_E_NOMEM paths.
namespace {
std::mutex g_alloc_mu;
int g_alloc_skip = 0, g_alloc_fail = 0;
}

cudaError_t lib_malloc(void **p, size_t bytes) {
    {
        std::lock_guard<std::mutex> lock(g_alloc_mu);
        if (g_alloc_skip > 0) {
            --g_alloc_skip;
        } else if (g_alloc_fail > 0) {
            --g_alloc_fail;
            *p = nullptr;
            return cudaErrorMemoryAllocation;
        }
    }
    return cudaMalloc(p, bytes);
}

// Cache buffers carry guard bands of a known byte on both sides; a kernel
// that writes outside its buffer changes them (rtr_*_check_guards).
constexpr size_t kGuardBytes = 64u << 10;
constexpr int kGuardByte = 0xA5;

char *guarded_alloc(size_t bytes) {
    void *raw = nullptr;
    if (lib_malloc(&raw, bytes + 2 * kGuardBytes) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    char *p = static_cast<char *>(raw) + kGuardBytes;
    if (cudaMemset(raw, kGuardByte, kGuardBytes) != cudaSuccess ||
        cudaMemset(p + bytes, kGuardByte, kGuardBytes) != cudaSuccess) {
        cudaFree(raw);
        return nullptr;
    }
    return p;
}

void guarded_free(char *p) {
    if (p) cudaFree(p - kGuardBytes);
}

// RTR_OK if both guard bands still hold kGuardByte (synchronises the device).
rtr_status guards_status(const char *p, size_t bytes) {
    if (cudaDeviceSynchronize() != cudaSuccess) return RTR_E_CUDA;
    std::vector<unsigned char> h(kGuardBytes);
    for (const char *g : {p - kGuardBytes, p + bytes}) {
        if (cudaMemcpy(h.data(), g, kGuardBytes, cudaMemcpyDeviceToHost) != cudaSuccess) return RTR_E_CUDA;
        for (unsigned char b : h)
            if (b != (unsigned char)kGuardByte) return RTR_E_STATE;
    }
    return RTR_OK;
}

bool shape_ok(int heads, int head_dim) { return heads >= 1 && (head_dim == 64 || head_dim == 128); }

float resolve_scale(float scale, int head_dim) { return scale > 0.f ? scale : 1.f / std::sqrt((float)head_dim); }

int sm_count(int device) {
    static std::atomic<int> cache[64] = {};
    if (device < 0 || device >= 64) return 148;
    int n = cache[device].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[device].store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace rtr

using namespace rtr;

// ------------------------------------------------------------------ handles
struct rtr_kvcache {
    int layers, heads, head_dim, k, R, W;
    int S;                   // physical window slots: W + commit room
    rtr_dtype dt;
    int device;
    long long rows;          // (R + S) * k rows per head
    size_t layer_bytes;      // heads * rows * head_dim * elt
    char *kbuf = nullptr, *vbuf = nullptr;
    std::vector<int> ref_valid, count;
    std::vector<long long> g;
    std::vector<CUtensorMap> tmk, tmv;
    std::vector<CUtensorMap> tmk64;   // K maps with 64-row boxes (CTA-pair attention)
    // Store maps of the fused cache writes, device array [layer][R + S][K, V][128-row, 8-row box]:
    // entry j covers row block j of a head (the reference frames, then the ring slots); bf16
    // caches with k a multiple of 8, else null.
    CUtensorMap *cmaps = nullptr;
};

struct rtr_xattn {
    int layers, heads, head_dim, max_text;
    rtr_dtype dt;
    int device;
    size_t layer_bytes;
    char *kbuf = nullptr, *vbuf = nullptr;
    std::vector<int> n_text;
    std::vector<CUtensorMap> tmk, tmv;
    std::vector<CUtensorMap> tmk64;   // K maps with 64-row boxes (CTA-pair attention)
};

namespace {

rtr_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return RTR_OK;
    if (e == cudaErrorMemoryAllocation) return RTR_E_NOMEM;
    return RTR_E_CUDA;
}

// Scratch buffers, one per (device, stream, slot) so that calls on different
// streams never share one: slot 0 holds the partial results of split
// attention units, slot 1 the DiT block's activations.  Grown on demand
// (cudaFree synchronises the device, so no kernel still uses the old buffer).
// A device keeps the buffers of its kMaxWorkspaceStreams most recently used
// (stream, slot) pairs: a caller that cycles through short-lived streams
// does not accumulate one buffer per stream.  The least recently used one is
// freed after a device synchronisation, so no kernel still reads it.
// rtr_release_workspaces frees a device's buffers on request.
constexpr size_t kMaxWorkspaceStreams = 8;

struct Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
    unsigned long long last_use = 0;
};

std::mutex g_ws_mu;
std::map<std::tuple<int, cudaStream_t, int>, Workspace> g_ws;
unsigned long long g_ws_clock = 0;

void *stream_workspace(int device, cudaStream_t s, size_t bytes, int slot = 0) {
    std::lock_guard<std::mutex> lock(g_ws_mu);
    const auto key = std::make_tuple(device, s, slot);
    auto it = g_ws.find(key);
    if (it == g_ws.end()) {
        size_t on_device = 0;
        auto lru = g_ws.end();
        for (auto j = g_ws.begin(); j != g_ws.end(); ++j) {
            if (std::get<0>(j->first) != device) continue;
            ++on_device;
            if (lru == g_ws.end() || j->second.last_use < lru->second.last_use) lru = j;
        }
        if (on_device >= kMaxWorkspaceStreams && lru != g_ws.end()) {
            if (cudaDeviceSynchronize() != cudaSuccess) return nullptr;
            if (lru->second.ptr) cudaFree(lru->second.ptr);
            g_ws.erase(lru);
        }
        it = g_ws.emplace(key, Workspace()).first;
    }
    Workspace &w = it->second;
    w.last_use = ++g_ws_clock;
    if (w.bytes < bytes) {
        if (w.ptr) cudaFree(w.ptr);
        w.ptr = nullptr;
        w.bytes = 0;
        if (lib_malloc(&w.ptr, bytes) != cudaSuccess) {
            cudaGetLastError();
            w.ptr = nullptr;
            return nullptr;
        }
        w.bytes = bytes;
    }
    return w.ptr;
}

// Frees every scratch buffer of `device` (the device is current).
rtr_status release_workspaces(int device) {
    std::lock_guard<std::mutex> lock(g_ws_mu);
    if (cudaDeviceSynchronize() != cudaSuccess) return RTR_E_CUDA;
    for (auto j = g_ws.begin(); j != g_ws.end();) {
        if (std::get<0>(j->first) == device) {
            if (j->second.ptr) cudaFree(j->second.ptr);
            j = g_ws.erase(j);
        } else {
            ++j;
        }
    }
    return RTR_OK;
}

size_t workspace_count(int device) {
    std::lock_guard<std::mutex> lock(g_ws_mu);
    size_t n = 0;
    for (auto &x : g_ws)
        if (std::get<0>(x.first) == device) ++n;
    return n;
}

// Launch the attention for a problem; picks the kernel for the element type.
// cta_group: 1 (one CTA per MMA, the default everywhere) or 2 (the CTA-pair
// kernel, reached only through rtr_attn_block_causal_prefill_ex).
rtr_status run_attention(AttnProblem &pb, rtr_dtype dt, const CUtensorMap *tm_k0, const CUtensorMap *tm_k0h,
                         const CUtensorMap *tm_v0, int device, cudaStream_t s, int cta_group = 1) {
    if (pb.nq == 0) return RTR_OK;
    for (int i = 0; i < pb.nseg; ++i)
        if (pb.seg[i].len <= 0) return RTR_E_INVAL;
    if (pb.nseg < 1) return RTR_E_INVAL;
    cudaError_t e;
    if (dt == RTR_BF16) {
        unsigned *st = device_status_ptr(device);
        if (!st) return RTR_E_CUDA;
        AttnPlan plan;
        // The chunk write (commit) is implemented for one CTA per MMA.
        plan_attn_bf16(pb, sm_count(device), pb.commit_k ? 1 : cta_group, plan);
        void *scratch = stream_workspace(device, s, plan.scratch_bytes);
        if (!scratch) return RTR_E_NOMEM;
        e = launch_attn_bf16(pb, plan, tm_k0, tm_k0h, tm_v0, st, scratch, s);
    } else {
        e = launch_attn_f32(pb, s);
    }
    return cuda_status(e);
}

}  // namespace

extern "C" {

const char *rtr_status_string(rtr_status s) {
    switch (s) {
        case RTR_OK: return "RTR_OK";
        case RTR_E_INVAL: return "RTR_E_INVAL: invalid argument";
        case RTR_E_NOMEM: return "RTR_E_NOMEM: device allocation failed";
        case RTR_E_STATE: return "RTR_E_STATE: call not valid in the current state";
        case RTR_E_CUDA: return "RTR_E_CUDA: CUDA call failed";
        case RTR_E_TIMEOUT: return "RTR_E_TIMEOUT: a kernel's bounded wait expired";
        case RTR_E_UNSUPPORTED: return "RTR_E_UNSUPPORTED: not implemented";
    }
    return "unknown rtr_status";
}

const char *rtr_build_info(void) {
    return "librtr: sm_100a tcgen05/TMEM/TMA frame-causal attention, fp32 CUDA-core path, "
           "vectorised KV-cache scatter";
}

rtr_status rtr_kvcache_create(int layers, int heads, int head_dim, int k, int ref_frames, int window_frames,
                              rtr_dtype dt, int device, rtr_kvcache **out) {
    return rtr_kvcache_create_ex(layers, heads, head_dim, k, ref_frames, window_frames, 0, dt, device, out);
}

rtr_status rtr_kvcache_create_ex(int layers, int heads, int head_dim, int k, int ref_frames, int window_frames,
                                 int commit_frames, rtr_dtype dt, int device, rtr_kvcache **out) {
    if (!out) return RTR_E_INVAL;
    *out = nullptr;
    if (layers < 1 || !shape_ok(heads, head_dim) || k < 1 || ref_frames < 0 || window_frames < 1 ||
        commit_frames < 0 || commit_frames > window_frames || (dt != RTR_BF16 && dt != RTR_F32) || device < 0)
        return RTR_E_INVAL;
    const long long rows = (long long)(ref_frames + window_frames + commit_frames) * k;
    if (rows > (1ll << 30) || (long long)heads * rows * head_dim >= (1ll << 40)) return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    rtr_kvcache *c = new (std::nothrow) rtr_kvcache();
    if (!c) return RTR_E_NOMEM;
    c->layers = layers; c->heads = heads; c->head_dim = head_dim; c->k = k;
    c->R = ref_frames; c->W = window_frames; c->S = window_frames + commit_frames;
    c->dt = dt; c->device = device;
    c->rows = rows;
    c->layer_bytes = (size_t)heads * rows * head_dim * elt_size(dt);
    const size_t total = c->layer_bytes * layers;
    c->kbuf = guarded_alloc(total);
    c->vbuf = c->kbuf ? guarded_alloc(total) : nullptr;
    if (!c->kbuf || !c->vbuf) {
        guarded_free(c->kbuf);
        delete c;
        return RTR_E_NOMEM;
    }
    if (cudaMemset(c->kbuf, 0, total) != cudaSuccess || cudaMemset(c->vbuf, 0, total) != cudaSuccess) {
        guarded_free(c->kbuf); guarded_free(c->vbuf); delete c;
        return RTR_E_CUDA;
    }
    c->ref_valid.assign(layers, 0);
    c->count.assign(layers, 0);
    c->g.assign(layers, 0);
    if (dt == RTR_BF16) {
        c->tmk.resize(layers);
        c->tmv.resize(layers);
        c->tmk64.resize(layers);
        for (int l = 0; l < layers; ++l) {
            if (!make_tmap_bf16(&c->tmk[l], c->kbuf + l * c->layer_bytes, head_dim, rows, heads, 128, 1) ||
                !make_tmap_bf16(&c->tmk64[l], c->kbuf + l * c->layer_bytes, head_dim, rows, heads, 64, 1) ||
                !make_tmap_bf16(&c->tmv[l], c->vbuf + l * c->layer_bytes, head_dim, rows, heads, 128, 1)) {
                guarded_free(c->kbuf); guarded_free(c->vbuf); delete c;
                return RTR_E_CUDA;
            }
        }
    }
    if (dt == RTR_BF16 && k % 8 == 0) {
        const int blocks = c->R + c->S;
        std::vector<CUtensorMap> maps((size_t)layers * blocks * 4);
        bool ok = true;
        const uint64_t row_bytes = (uint64_t)head_dim * 2;
        for (int l = 0; l < layers && ok; ++l)
            for (int j = 0; j < blocks && ok; ++j)
                for (int kv = 0; kv < 2 && ok; ++kv) {
                    const char *base = (kv ? c->vbuf : c->kbuf) + l * c->layer_bytes + (size_t)j * k * row_bytes;
                    CUtensorMap *m = &maps[(((size_t)l * blocks + j) * 2 + kv) * 2];
                    ok = make_tmap_bf16_strided(m, base, head_dim, k, heads, (uint64_t)rows * row_bytes, 128, 1) &&
                         make_tmap_bf16_strided(m + 1, base, head_dim, k, heads, (uint64_t)rows * row_bytes, 8, 1);
                }
        if (!ok || lib_malloc(reinterpret_cast<void **>(&c->cmaps), maps.size() * sizeof(CUtensorMap)) != cudaSuccess ||
            cudaMemcpy(c->cmaps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice) !=
                cudaSuccess) {
            cudaGetLastError();
            if (c->cmaps) cudaFree(c->cmaps);
            guarded_free(c->kbuf); guarded_free(c->vbuf); delete c;
            return ok ? RTR_E_NOMEM : RTR_E_CUDA;
        }
    }
    if (cudaDeviceSynchronize() != cudaSuccess) {
        if (c->cmaps) cudaFree(c->cmaps);
        guarded_free(c->kbuf); guarded_free(c->vbuf); delete c;
        return RTR_E_CUDA;
    }
    *out = c;
    return RTR_OK;
}

void rtr_kvcache_destroy(rtr_kvcache *c) {
    if (!c) return;
    DeviceGuard dg(c->device);
    cudaDeviceSynchronize();
    if (c->cmaps) cudaFree(c->cmaps);
    guarded_free(c->kbuf);
    guarded_free(c->vbuf);
    delete c;
}

rtr_status rtr_kvcache_set_reference(rtr_kvcache *c, int layer, const void *k_ref, const void *v_ref,
                                     rtr_stream_t stream) {
    if (!c || layer < 0 || layer >= c->layers || !aligned16(k_ref) || !aligned16(v_ref)) return RTR_E_INVAL;
    if (c->R == 0) return RTR_E_STATE;
    DeviceGuard dg(c->device);
    ScatterArgs a;
    a.src_k = k_ref; a.src_v = v_ref;
    a.dst_k = c->kbuf + layer * c->layer_bytes;
    a.dst_v = c->vbuf + layer * c->layer_bytes;
    a.n_tok = c->R * c->k; a.heads = c->heads; a.row_bytes = c->head_dim * (int)elt_size(c->dt);
    a.k_frame = c->k; a.first_slot = 0; a.slot_mod = c->R; a.slot_off = 0;
    a.rows_per_head = c->rows;
    rtr_status st = cuda_status(launch_kv_scatter(a, (cudaStream_t)stream));
    if (st == RTR_OK) c->ref_valid[layer] = 1;
    return st;
}

rtr_status rtr_kvcache_clear_reference(rtr_kvcache *c, int layer) {
    if (!c || layer < -1 || layer >= c->layers) return RTR_E_INVAL;
    for (int l = 0; l < c->layers; ++l)
        if (layer == -1 || l == layer) c->ref_valid[l] = 0;
    return RTR_OK;
}

rtr_status rtr_kvcache_append_frame(rtr_kvcache *c, int layer, const void *k_new, const void *v_new, int n_frames,
                                    rtr_stream_t stream) {
    if (!c || layer < 0 || layer >= c->layers || !aligned16(k_new) || !aligned16(v_new)) return RTR_E_INVAL;
    if (n_frames < 1 || n_frames > c->W) return RTR_E_INVAL;
    DeviceGuard dg(c->device);
    ScatterArgs a;
    a.src_k = k_new; a.src_v = v_new;
    a.dst_k = c->kbuf + layer * c->layer_bytes;
    a.dst_v = c->vbuf + layer * c->layer_bytes;
    a.n_tok = n_frames * c->k; a.heads = c->heads; a.row_bytes = c->head_dim * (int)elt_size(c->dt);
    a.k_frame = c->k; a.first_slot = (int)(c->g[layer] % c->S); a.slot_mod = c->S; a.slot_off = c->R;
    a.rows_per_head = c->rows;
    rtr_status st = cuda_status(launch_kv_scatter(a, (cudaStream_t)stream));
    if (st == RTR_OK) {
        c->g[layer] += n_frames;
        c->count[layer] = std::min(c->W, c->count[layer] + n_frames);
    }
    return st;
}

rtr_status rtr_kvcache_retain_last(rtr_kvcache *c, int layer, int n_frames) {
    if (!c || layer < -1 || layer >= c->layers || n_frames < 0) return RTR_E_INVAL;
    for (int l = 0; l < c->layers; ++l)
        if (layer == -1 || l == layer) c->count[l] = std::min(c->count[l], n_frames);
    return RTR_OK;
}

rtr_status rtr_kvcache_get_index_map(const rtr_kvcache *c, int layer, int32_t *slot_frame, int32_t *ref_valid,
                                     int64_t *frames_appended, int32_t *count) {
    if (!c || layer < 0 || layer >= c->layers) return RTR_E_INVAL;
    const long long g = c->g[layer];
    const int cnt = c->count[layer];
    if (slot_frame) {
        for (int s = 0; s < c->S; ++s) slot_frame[s] = -1;
        for (long long f = g - cnt; f < g; ++f) slot_frame[f % c->S] = (int32_t)f;
    }
    if (ref_valid) *ref_valid = c->ref_valid[layer];
    if (frames_appended) *frames_appended = g;
    if (count) *count = cnt;
    return RTR_OK;
}

rtr_status rtr_kvcache_set_index_map(rtr_kvcache *c, int layer, int64_t frames_appended, int32_t count,
                                     int32_t ref_valid) {
    if (!c || layer < 0 || layer >= c->layers || frames_appended < 0 || count < 0 || count > c->W ||
        (int64_t)count > frames_appended || (ref_valid != 0 && ref_valid != 1) || (ref_valid && c->R == 0))
        return RTR_E_INVAL;
    c->g[layer] = frames_appended;
    c->count[layer] = count;
    c->ref_valid[layer] = ref_valid;
    return RTR_OK;
}

rtr_status rtr_kvcache_check_guards(const rtr_kvcache *c) {
    if (!c) return RTR_E_INVAL;
    DeviceGuard dg(c->device);
    const size_t total = c->layer_bytes * c->layers;
    const rtr_status a = guards_status(c->kbuf, total);
    return a != RTR_OK ? a : guards_status(c->vbuf, total);
}

rtr_status rtr_kvcache_device_ptrs(const rtr_kvcache *c, int layer, void **k, void **v) {
    if (!c || layer < 0 || layer >= c->layers || !k || !v) return RTR_E_INVAL;
    *k = c->kbuf + layer * c->layer_bytes;
    *v = c->vbuf + layer * c->layer_bytes;
    return RTR_OK;
}

namespace {

// The stream attention problem of one layer: key runs for the reference and
// the held window frames (physical order), then the chunk itself.
rtr_status stream_problem(const rtr_kvcache *c, int layer, const void *q, const void *k_cur, const void *v_cur,
                          int n_cur_frames, void *out, float scale, AttnProblem &pb) {
    if (!c || layer < 0 || layer >= c->layers || n_cur_frames < 1) return RTR_E_INVAL;
    if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(out)) return RTR_E_INVAL;
    const long long nq = (long long)n_cur_frames * c->k;
    if (nq > (1ll << 30)) return RTR_E_INVAL;
    // Physical row intervals of the cached keys: the reference slot and the
    // held window frames.  Every cached key is visible to every chunk query,
    // so adjacent intervals merge and their order is free.
    std::vector<std::pair<long long, long long>> iv;
    if (c->ref_valid[layer] && c->R > 0) iv.push_back({0, (long long)c->R * c->k});
    const long long g = c->g[layer];
    for (long long f = g - c->count[layer]; f < g; ++f) {
        const long long s = f % c->S;
        iv.push_back({(c->R + s) * c->k, (c->R + s + 1) * c->k});
    }
    std::sort(iv.begin(), iv.end());
    std::vector<std::pair<long long, long long>> merged;
    for (auto &x : iv) {
        if (!merged.empty() && merged.back().second == x.first)
            merged.back().second = x.second;
        else
            merged.push_back(x);
    }
    if (merged.size() > (size_t)kMaxSegs - 1) return RTR_E_UNSUPPORTED;   // cannot happen: <= 3 runs
    memset(&pb, 0, sizeof(pb));
    pb.nq = (int)nq; pb.heads = c->heads; pb.head_dim = c->head_dim; pb.kpf = c->k;
    // The chunk's run goes last, so that every unit of a head sweeps the
    // cached keys in step with the others (they share them through L2).  The
    // fused commit uses the same order, so its outputs are bit-identical to
    // attention + append on the same cache.
    for (auto &x : merged) pb.seg[pb.nseg++] = KvSeg{0, (int)x.first, (int)(x.second - x.first), 0};
    pb.seg[pb.nseg++] = KvSeg{1, 0, (int)nq, 1};
    pb.scale = resolve_scale(scale, c->head_dim);
    pb.q = q; pb.o = out;
    pb.k0 = c->kbuf + layer * c->layer_bytes; pb.v0 = c->vbuf + layer * c->layer_bytes; pb.rows0 = c->rows;
    pb.k1 = k_cur; pb.v1 = v_cur; pb.rows1 = nq;
    return RTR_OK;
}

}  // namespace

rtr_status rtr_attn_frame_causal(const rtr_kvcache *c, int layer, const void *q, const void *k_cur,
                                 const void *v_cur, int n_cur_frames, void *out, float scale, rtr_stream_t stream) {
    return rtr_attn_frame_causal_ex(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale, 1, stream);
}

rtr_status rtr_attn_frame_causal_ex(const rtr_kvcache *c, int layer, const void *q, const void *k_cur,
                                    const void *v_cur, int n_cur_frames, void *out, float scale, int cta_group,
                                    rtr_stream_t stream) {
    if (cta_group != 1 && cta_group != 2) return RTR_E_INVAL;
    AttnProblem pb;
    const rtr_status st = stream_problem(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale, pb);
    if (st != RTR_OK) return st;
    DeviceGuard dg(c->device);
    const CUtensorMap *tk = c->dt == RTR_BF16 ? &c->tmk[layer] : nullptr;
    const CUtensorMap *tkh = c->dt == RTR_BF16 ? &c->tmk64[layer] : nullptr;
    const CUtensorMap *tv = c->dt == RTR_BF16 ? &c->tmv[layer] : nullptr;
    return run_attention(pb, c->dt, tk, tkh, tv, c->device, (cudaStream_t)stream, cta_group);
}

rtr_status rtr_attn_frame_causal_f32out(const rtr_kvcache *c, int layer, const void *q, const void *k_cur,
                                        const void *v_cur, int n_cur_frames, float *out, float scale,
                                        rtr_stream_t stream) {
    if (c && c->dt == RTR_F32)   // the fp32 path's output is fp32 already
        return rtr_attn_frame_causal_ex(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale, 1, stream);
    AttnProblem pb;
    const rtr_status st = stream_problem(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale, pb);
    if (st != RTR_OK) return st;
    pb.o_f32 = out;
    pb.o = nullptr;
    DeviceGuard dg(c->device);
    return run_attention(pb, c->dt, &c->tmk[layer], &c->tmk64[layer], &c->tmv[layer], c->device,
                         (cudaStream_t)stream, 1);
}

rtr_status rtr_attn_frame_causal_commit(rtr_kvcache *c, int layer, const void *q, const void *k_cur,
                                        const void *v_cur, int n_cur_frames, void *out, float scale,
                                        rtr_stream_t stream) {
    AttnProblem pb;
    const rtr_status st = stream_problem(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale, pb);
    if (st != RTR_OK) return st;
    // The chunk's frames go to slots the held window does not use.
    if (n_cur_frames > c->S - c->W) return RTR_E_INVAL;
    DeviceGuard dg(c->device);
    if (c->dt != RTR_BF16) {
        // fp32 storage: the attention kernel, then the scatter kernel.
        rtr_status r = run_attention(pb, c->dt, nullptr, nullptr, nullptr, c->device, (cudaStream_t)stream);
        if (r != RTR_OK) return r;
        return rtr_kvcache_append_frame(c, layer, k_cur, v_cur, n_cur_frames, stream);
    }
    pb.commit_k = c->kbuf + layer * c->layer_bytes;
    pb.commit_v = c->vbuf + layer * c->layer_bytes;
    pb.commit_first_slot = (int)(c->g[layer] % c->S);
    pb.commit_slots = c->S;
    pb.commit_row0 = c->R * c->k;
    pb.commit_maps = c->cmaps ? c->cmaps + ((size_t)layer * (c->R + c->S) + c->R) * 4 : nullptr;
    const rtr_status r = run_attention(pb, c->dt, &c->tmk[layer], &c->tmk64[layer], &c->tmv[layer], c->device,
                                       (cudaStream_t)stream);
    if (r == RTR_OK) {
        c->g[layer] += n_cur_frames;
        c->count[layer] = std::min(c->W, c->count[layer] + n_cur_frames);
    }
    return r;
}

rtr_status rtr_attn_block_causal_prefill(const void *q, const void *k, const void *v, int n_tokens, int heads,
                                         int head_dim, int k_per_frame, rtr_dtype dt, void *out, float scale,
                                         int device, rtr_stream_t stream) {
    return rtr_attn_block_causal_prefill_ex(q, k, v, n_tokens, heads, head_dim, k_per_frame, dt, out, scale, 1,
                                            device, stream);
}

rtr_status rtr_attn_block_causal_prefill_ex(const void *q, const void *k, const void *v, int n_tokens, int heads,
                                            int head_dim, int k_per_frame, rtr_dtype dt, void *out, float scale,
                                            int cta_group, int device, rtr_stream_t stream) {
    if (n_tokens < 0 || !shape_ok(heads, head_dim) || k_per_frame < 1 || (dt != RTR_BF16 && dt != RTR_F32) ||
        device < 0 || (cta_group != 1 && cta_group != 2))
        return RTR_E_INVAL;
    if (n_tokens == 0) return RTR_OK;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return RTR_E_INVAL;
    if (n_tokens > (1 << 30)) return RTR_E_INVAL;
    AttnProblem pb;
    memset(&pb, 0, sizeof(pb));
    pb.nq = n_tokens; pb.heads = heads; pb.head_dim = head_dim; pb.kpf = k_per_frame;
    pb.nseg = 1;
    pb.seg[0] = KvSeg{1, 0, n_tokens, 1};
    pb.scale = resolve_scale(scale, head_dim);
    pb.q = q; pb.o = out; pb.k1 = k; pb.v1 = v; pb.rows1 = n_tokens;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    return run_attention(pb, dt, nullptr, nullptr, nullptr, device, (cudaStream_t)stream, cta_group);
}

rtr_status rtr_attn_block_causal_prefill_lse(const void *q, const void *k, const void *v, int n_tokens, int heads,
                                             int head_dim, int k_per_frame, rtr_dtype dt, void *out, float *lse,
                                             float scale, int device, rtr_stream_t stream) {
    if (n_tokens < 0 || !shape_ok(heads, head_dim) || k_per_frame < 1 || (dt != RTR_BF16 && dt != RTR_F32) ||
        device < 0)
        return RTR_E_INVAL;
    if (dt != RTR_BF16) return RTR_E_UNSUPPORTED;
    if (n_tokens == 0) return RTR_OK;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !lse) return RTR_E_INVAL;
    if (n_tokens > (1 << 30)) return RTR_E_INVAL;
    AttnProblem pb;
    memset(&pb, 0, sizeof(pb));
    pb.nq = n_tokens; pb.heads = heads; pb.head_dim = head_dim; pb.kpf = k_per_frame;
    pb.nseg = 1;
    pb.seg[0] = KvSeg{1, 0, n_tokens, 1};
    pb.scale = resolve_scale(scale, head_dim);
    pb.q = q; pb.o = out; pb.k1 = k; pb.v1 = v; pb.rows1 = n_tokens;
    pb.lse = lse;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    return run_attention(pb, dt, nullptr, nullptr, nullptr, device, (cudaStream_t)stream);
}

rtr_status rtr_attn_block_causal_prefill_cache(rtr_kvcache *c, int layer, const void *q, const void *k,
                                               const void *v, int n_frames, int with_reference, void *out,
                                               float scale, rtr_stream_t stream) {
    if (!c || layer < 0 || layer >= c->layers || n_frames < 1 || (with_reference != 0 && with_reference != 1))
        return RTR_E_INVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return RTR_E_INVAL;
    if (with_reference && c->R == 0) return RTR_E_STATE;
    const int nref = with_reference ? c->R : 0;
    const int nwin = n_frames - nref;
    if (nwin < 0 || nwin > c->W) return RTR_E_INVAL;
    const long long n = (long long)n_frames * c->k;
    if (n > (1ll << 30)) return RTR_E_INVAL;
    DeviceGuard dg(c->device);
    AttnProblem pb;
    memset(&pb, 0, sizeof(pb));
    pb.nq = (int)n; pb.heads = c->heads; pb.head_dim = c->head_dim; pb.kpf = c->k;
    pb.nseg = 1;
    pb.seg[0] = KvSeg{1, 0, (int)n, 1};
    pb.scale = resolve_scale(scale, c->head_dim);
    pb.q = q; pb.o = out; pb.k1 = k; pb.v1 = v; pb.rows1 = n;
    pb.rows0 = c->rows;
    const long long g = c->g[layer];
    // One launch writes the sequence's K/V while it attends when every frame's
    // rows follow from one slot rule: without a reference part the frames are
    // appended to the ring (slot (g + i) mod S); with one, the reference frames
    // and the ring slots form one run of row blocks when g is a multiple of S.
    if (c->dt == RTR_BF16 && (nref == 0 || g % c->S == 0)) {
        pb.commit_k = c->kbuf + layer * c->layer_bytes;
        pb.commit_v = c->vbuf + layer * c->layer_bytes;
        const size_t maps0 = (size_t)layer * (c->R + c->S);
        if (nref > 0) {
            pb.commit_row0 = 0;
            pb.commit_slots = c->R + c->S;
            pb.commit_first_slot = 0;
            pb.commit_maps = c->cmaps ? c->cmaps + maps0 * 4 : nullptr;
        } else {
            pb.commit_row0 = c->R * c->k;
            pb.commit_slots = c->S;
            pb.commit_first_slot = (int)(g % c->S);
            pb.commit_maps = c->cmaps ? c->cmaps + (maps0 + c->R) * 4 : nullptr;
        }
        const rtr_status r = run_attention(pb, c->dt, nullptr, nullptr, nullptr, c->device, (cudaStream_t)stream);
        if (r != RTR_OK) return r;
        if (nref > 0) c->ref_valid[layer] = 1;
        if (nwin > 0) {
            c->g[layer] += nwin;
            c->count[layer] = std::min(c->W, c->count[layer] + nwin);
        }
        return RTR_OK;
    }
    // Otherwise (fp32 storage, or a reference part with g not a multiple of
    // S): the attention, then the copy kernels of set_reference and append.
    rtr_status r = run_attention(pb, c->dt, nullptr, nullptr, nullptr, c->device, (cudaStream_t)stream);
    if (r != RTR_OK) return r;
    const size_t frame_bytes = (size_t)c->k * c->heads * c->head_dim * elt_size(c->dt);
    if (nref > 0) {
        r = rtr_kvcache_set_reference(c, layer, k, v, stream);
        if (r != RTR_OK) return r;
    }
    if (nwin > 0)
        r = rtr_kvcache_append_frame(c, layer, static_cast<const char *>(k) + nref * frame_bytes,
                                     static_cast<const char *>(v) + nref * frame_bytes, nwin, stream);
    return r;
}

rtr_status rtr_attn_block_causal_backward(const void *q, const void *k, const void *v, const void *out,
                                          const void *dout, const float *lse, int n_tokens, int heads,
                                          int head_dim, int k_per_frame, rtr_dtype dt, void *dq, void *dk,
                                          void *dv, float scale, int device, rtr_stream_t stream) {
    if (n_tokens < 0 || !shape_ok(heads, head_dim) || k_per_frame < 1 || (dt != RTR_BF16 && dt != RTR_F32) ||
        device < 0)
        return RTR_E_INVAL;
    if (dt != RTR_BF16) return RTR_E_UNSUPPORTED;
    if (n_tokens == 0) return RTR_OK;
    for (const void *ptr : {q, k, v, out, dout, (const void *)dq, (const void *)dk, (const void *)dv})
        if (!aligned16(ptr)) return RTR_E_INVAL;
    if (!lse || n_tokens > (1 << 30)) return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    unsigned *st = device_status_ptr(device);
    if (!st) return RTR_E_CUDA;
    void *scratch = stream_workspace(device, (cudaStream_t)stream, bwd_scratch_bytes(n_tokens, heads));
    if (!scratch) return RTR_E_NOMEM;
    BwdProblem pb;
    pb.q = q; pb.k = k; pb.v = v; pb.o = out; pb.dout = dout; pb.lse = lse;
    pb.dq = dq; pb.dk = dk; pb.dv = dv;
    pb.n = n_tokens; pb.heads = heads; pb.head_dim = head_dim; pb.kpf = k_per_frame;
    pb.scale = resolve_scale(scale, head_dim);
    return cuda_status(launch_attn_bwd(pb, st, scratch, (cudaStream_t)stream));
}

}  // extern "C"

namespace {

// The block's weights as the projections read them: each matrix either
// row-major [in][out] or in the packed B layout.
struct DitW {
    const void *wqkv, *wo, *wq2, *wo2, *w1, *w2;
    const void *bqkv, *bo, *bq2, *bo2, *b1, *b2;
    int d_ffn;
    int packed;
};

rtr_status dit_block_run(rtr_kvcache *c, const rtr_xattn *x, int layer, const DitW &w, const void *modulation,
                         void *hidden, int n_cur_frames, int grid_h, int grid_w, int t0, int commit,
                         rtr_stream_t stream) {
    if (!c || !x || layer < 0 || layer >= c->layers || layer >= x->layers || n_cur_frames < 1 || grid_h < 1 ||
        grid_w < 1 || t0 < 0 || (commit != 0 && commit != 1))
        return RTR_E_INVAL;
    if (c->dt != RTR_BF16 || x->dt != RTR_BF16 || x->heads != c->heads || x->head_dim != c->head_dim ||
        x->device != c->device || (long long)grid_h * grid_w != c->k)
        return RTR_E_INVAL;
    const int H = c->heads, d = c->head_dim, D = H * d, F = w.d_ffn;
    if (F < 8 || F % 8 != 0 || (commit && n_cur_frames > c->W)) return RTR_E_INVAL;
    for (const void *ptr : {modulation, (const void *)hidden, w.wqkv, w.bqkv, w.wo, w.bo, w.wq2, w.bq2, w.wo2, w.bo2,
                            w.w1, w.b1, w.w2, w.b2})
        if (!aligned16(ptr)) return RTR_E_INVAL;
    const long long n = (long long)n_cur_frames * c->k;
    if (n > (1 << 24)) return RTR_E_INVAL;
    if (x->n_text[layer] == 0) return RTR_E_STATE;
    DeviceGuard dg(c->device);
    const cudaStream_t s = (cudaStream_t)stream;
    unsigned *status = device_status_ptr(c->device);
    if (!status) return RTR_E_CUDA;
    const int sms = sm_count(c->device);
    // Activations: q, k, v, o (bf16 [n][D]); the layer-norm output h, the
    // projections' A operand, in the packed layout (D is a multiple of 64);
    // the GELU output f, the last projection's A operand, packed when F is a
    // multiple of 64, else [n][F].
    const int f_packed = F % 64 == 0;
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    const size_t nd = up((size_t)n * D * 2), nh = up(packed_a_bytes(n, D));
    const size_t nf = up(f_packed ? packed_a_bytes(n, F) : (size_t)n * F * 2);
    char *ws = static_cast<char *>(stream_workspace(c->device, s, nh + 4 * nd + nf, 1));
    if (!ws) return RTR_E_NOMEM;
    void *h = ws, *q = ws + nh, *k = ws + nh + nd, *v = ws + nh + 2 * nd, *o = ws + nh + 3 * nd,
         *f = ws + nh + 4 * nd;
    const char *mod = static_cast<const char *>(modulation);
    const size_t mrow = (size_t)D * 2;   // one modulation vector, bytes
    const int ni = (int)n;
    const float eps = 1e-6f;
    cudaError_t e = cudaSuccess;
    rtr_status st = RTR_OK;
    // One projection with its epilogue: a = activations [n][in] (packed when
    // a_packed), wt = [in][out] weights (packed when w.packed).
    auto gemm = [&](const void *a, int a_packed, const void *wt, int n_out, int n_in, int epi, const void *bias,
                    const void *gate, void *out, int out_packed) {
        GemmArgs g;
        memset(&g, 0, sizeof(g));
        g.a = a; g.w = wt; g.m = ni; g.n = n_out; g.k = n_in; g.epi = epi;
        g.a_packed = a_packed; g.w_packed = w.packed; g.out_packed = out_packed;
        g.bias = bias; g.gate = gate; g.out = out;
        if (epi == kEpiQkvRope) {
            g.q = q; g.k_out = k; g.v = v;
            g.head_dim = d; g.kpf = c->k; g.grid_w = grid_w; g.t0 = t0;
        }
        return launch_gemm_bf16(g, status, sms, s);
    };
#define RTR_TRY(call)                                   \
    do {                                                \
        if ((e = (call)) != cudaSuccess) return cuda_status(e); \
    } while (0)
#define RTR_TRY_ST(call)                                \
    do {                                                \
        if ((st = (call)) != RTR_OK) return st;         \
    } while (0)
    // self attention branch
    RTR_TRY(launch_ln_modulate(hidden, mod, mod + mrow, h, ni, D, eps, s, 1));
    RTR_TRY(gemm(h, 1, w.wqkv, 3 * D, D, kEpiQkvRope, w.bqkv, nullptr, nullptr, 0));
    if (commit && c->S - c->W >= n_cur_frames) {
        RTR_TRY_ST(rtr_attn_frame_causal_commit(c, layer, q, k, v, n_cur_frames, o, 0.f, stream));
    } else {
        RTR_TRY_ST(rtr_attn_frame_causal(c, layer, q, k, v, n_cur_frames, o, 0.f, stream));
        if (commit) RTR_TRY_ST(rtr_kvcache_append_frame(c, layer, k, v, n_cur_frames, stream));
    }
    RTR_TRY(gemm(o, 0, w.wo, D, D, kEpiGatedResidual, w.bo, mod + 2 * mrow, hidden, 0));
    // cross attention branch
    RTR_TRY(launch_ln_modulate(hidden, nullptr, nullptr, h, ni, D, eps, s, 1));
    RTR_TRY(gemm(h, 1, w.wq2, D, D, kEpiBias, w.bq2, nullptr, q, 0));
    RTR_TRY_ST(rtr_attn_cross(x, layer, q, ni, o, 0.f, stream));
    RTR_TRY(gemm(o, 0, w.wo2, D, D, kEpiGatedResidual, w.bo2, nullptr, hidden, 0));
    // feed-forward branch
    RTR_TRY(launch_ln_modulate(hidden, mod + 3 * mrow, mod + 4 * mrow, h, ni, D, eps, s, 1));
    RTR_TRY(gemm(h, 1, w.w1, F, D, kEpiBiasGelu, w.b1, nullptr, f, f_packed));
    RTR_TRY(gemm(f, f_packed, w.w2, D, F, kEpiGatedResidual, w.b2, mod + 5 * mrow, hidden, 0));
#undef RTR_TRY
#undef RTR_TRY_ST
    return RTR_OK;
}

}  // namespace

struct rtr_dit_packed {
    int device, d_model, d_ffn;
    char *buf = nullptr;   // the six packed matrices, then copies of the six biases
    DitW w;
};

extern "C" {

rtr_status rtr_dit_block_forward(rtr_kvcache *c, const rtr_xattn *x, int layer, const rtr_dit_weights *w,
                                 const void *modulation, void *hidden, int n_cur_frames, int grid_h, int grid_w,
                                 int t0, int commit, rtr_stream_t stream) {
    if (!w) return RTR_E_INVAL;
    DitW dw = {w->wqkv, w->wo, w->wq2, w->wo2, w->w1, w->w2, w->bqkv, w->bo, w->bq2, w->bo2, w->b1, w->b2,
               w->d_ffn, 0};
    return dit_block_run(c, x, layer, dw, modulation, hidden, n_cur_frames, grid_h, grid_w, t0, commit, stream);
}

rtr_status rtr_dit_block_forward_packed(rtr_kvcache *c, const rtr_xattn *x, int layer, const rtr_dit_packed *pw,
                                        const void *modulation, void *hidden, int n_cur_frames, int grid_h,
                                        int grid_w, int t0, int commit, rtr_stream_t stream) {
    if (!pw || !c || pw->device != c->device || pw->d_model != c->heads * c->head_dim) return RTR_E_INVAL;
    return dit_block_run(c, x, layer, pw->w, modulation, hidden, n_cur_frames, grid_h, grid_w, t0, commit, stream);
}

rtr_status rtr_dit_pack_weights(const rtr_dit_weights *w, int d_model, int device, rtr_stream_t stream,
                                rtr_dit_packed **out) {
    if (!out) return RTR_E_INVAL;
    *out = nullptr;
    if (!w || device < 0 || d_model < 64 || d_model % 64 != 0 || w->d_ffn < 64 || w->d_ffn % 64 != 0)
        return RTR_E_INVAL;
    for (const void *ptr : {w->wqkv, w->bqkv, w->wo, w->bo, w->wq2, w->bq2, w->wo2, w->bo2, w->w1, w->b1, w->w2,
                            w->b2})
        if (!aligned16(ptr)) return RTR_E_INVAL;
    const int D = d_model, F = w->d_ffn;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    const cudaStream_t s = (cudaStream_t)stream;
    // matrices (k, n) and biases (length) in buffer order
    const int mk[6] = {D, D, D, D, D, F}, mn[6] = {3 * D, D, D, D, F, D};
    const void *msrc[6] = {w->wqkv, w->wo, w->wq2, w->wo2, w->w1, w->w2};
    const void *bsrc[6] = {w->bqkv, w->bo, w->bq2, w->bo2, w->b1, w->b2};
    size_t off[12], total = 0;
    for (int i = 0; i < 6; ++i) {
        off[i] = total;
        total += (packed_b_bytes(mk[i], mn[i]) + 255) & ~size_t(255);
    }
    for (int i = 0; i < 6; ++i) {
        off[6 + i] = total;
        total += ((size_t)mn[i] * 2 + 255) & ~size_t(255);
    }
    rtr_dit_packed *pw = new (std::nothrow) rtr_dit_packed();
    if (!pw) return RTR_E_NOMEM;
    void *raw = nullptr;
    if (lib_malloc(&raw, total) != cudaSuccess) {
        cudaGetLastError();
        delete pw;
        return RTR_E_NOMEM;
    }
    pw->buf = static_cast<char *>(raw);
    pw->device = device;
    pw->d_model = D;
    pw->d_ffn = F;
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 6 && e == cudaSuccess; ++i) e = launch_pack_b(msrc[i], pw->buf + off[i], mk[i], mn[i], s);
    for (int i = 0; i < 6 && e == cudaSuccess; ++i)
        e = cudaMemcpyAsync(pw->buf + off[6 + i], bsrc[i], (size_t)mn[i] * 2, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        cudaFree(pw->buf);
        delete pw;
        return RTR_E_CUDA;
    }
    const char *b = pw->buf;
    pw->w = DitW{b + off[0], b + off[1], b + off[2], b + off[3], b + off[4], b + off[5],
                 b + off[6], b + off[7], b + off[8], b + off[9], b + off[10], b + off[11], F, 1};
    *out = pw;
    return RTR_OK;
}

void rtr_dit_packed_destroy(rtr_dit_packed *pw) {
    if (!pw) return;
    DeviceGuard dg(pw->device);
    cudaDeviceSynchronize();
    cudaFree(pw->buf);
    delete pw;
}

rtr_status rtr_dit_linear(const void *a, const void *w, int m, int n, int k, rtr_epilogue epilogue, const void *bias,
                          const void *gate, void *out, int device, rtr_stream_t stream) {
    if (m < 0 || n < 8 || k < 8 || n % 8 != 0 || k % 8 != 0 || device < 0 ||
        (epilogue != RTR_EPI_BIAS && epilogue != RTR_EPI_BIAS_GELU && epilogue != RTR_EPI_GATED_RESIDUAL))
        return RTR_E_INVAL;
    if (m == 0) return RTR_OK;
    if (!aligned16(a) || !aligned16(w) || !aligned16(bias) || !aligned16(out) || (gate && !aligned16(gate)) ||
        (gate && epilogue != RTR_EPI_GATED_RESIDUAL))
        return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    unsigned *status = device_status_ptr(device);
    if (!status) return RTR_E_CUDA;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.a = a; g.w = w; g.m = m; g.n = n; g.k = k;
    g.epi = epilogue == RTR_EPI_BIAS ? kEpiBias : epilogue == RTR_EPI_BIAS_GELU ? kEpiBiasGelu : kEpiGatedResidual;
    g.bias = bias; g.gate = gate; g.out = out;
    return cuda_status(launch_gemm_bf16(g, status, sm_count(device), (cudaStream_t)stream));
}

rtr_status rtr_dit_qkv_rope(const void *a, const void *wqkv, const void *bqkv, int m, int d_in, int heads,
                            int head_dim, int k_per_frame, int grid_w, int t0, void *q, void *k, void *v, int device,
                            rtr_stream_t stream) {
    if (m < 0 || d_in < 8 || d_in % 8 != 0 || !shape_ok(heads, head_dim) || k_per_frame < 1 || grid_w < 1 ||
        t0 < 0 || device < 0)
        return RTR_E_INVAL;
    if (m == 0) return RTR_OK;
    for (const void *ptr : {a, wqkv, bqkv, (const void *)q, (const void *)k, (const void *)v})
        if (!aligned16(ptr)) return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    unsigned *status = device_status_ptr(device);
    if (!status) return RTR_E_CUDA;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.a = a; g.w = wqkv; g.m = m; g.n = 3 * heads * head_dim; g.k = d_in; g.epi = kEpiQkvRope;
    g.bias = bqkv; g.q = q; g.k_out = k; g.v = v;
    g.head_dim = head_dim; g.kpf = k_per_frame; g.grid_w = grid_w; g.t0 = t0;
    return cuda_status(launch_gemm_bf16(g, status, sm_count(device), (cudaStream_t)stream));
}

rtr_status rtr_dit_linear_tile(int m, int n, int k, rtr_epilogue epilogue, int qkv_rope, int device, int *rows,
                               int *cols, int *cta_pair, int *ctas) {
    if (m < 1 || n < 1 || k < 1 || device < 0 || !rows || !cols || !cta_pair || !ctas ||
        (epilogue != RTR_EPI_BIAS && epilogue != RTR_EPI_BIAS_GELU && epilogue != RTR_EPI_GATED_RESIDUAL))
        return RTR_E_INVAL;
    const int epi = qkv_rope ? kEpiQkvRope
                    : epilogue == RTR_EPI_BIAS ? kEpiBias
                    : epilogue == RTR_EPI_BIAS_GELU ? kEpiBiasGelu : kEpiGatedResidual;
    DeviceGuard dg(device);
    gemm_tile_shape(m, n, k, epi, device, sm_count(device), rows, cols, cta_pair, ctas);
    return RTR_OK;
}

rtr_status rtr_dit_plan_tile(int m, int n, int k, rtr_epilogue epilogue, int qkv_rope, int w_packed, int sms,
                             int pair_clusters, int *rows, int *cols, int *cta_pair, int *ctas) {
    if (m < 1 || n < 1 || k < 1 || sms < 1 || pair_clusters < 0 || pair_clusters > sms / 2 || !rows || !cols ||
        !cta_pair || !ctas ||
        (epilogue != RTR_EPI_BIAS && epilogue != RTR_EPI_BIAS_GELU && epilogue != RTR_EPI_GATED_RESIDUAL))
        return RTR_E_INVAL;
    const int epi = qkv_rope ? kEpiQkvRope
                    : epilogue == RTR_EPI_BIAS ? kEpiBias
                    : epilogue == RTR_EPI_BIAS_GELU ? kEpiBiasGelu : kEpiGatedResidual;
    gemm_plan_tile(m, n, k, epi, w_packed != 0, sms, pair_clusters, rows, cols, cta_pair, ctas);
    return RTR_OK;
}

rtr_status rtr_crossattn_create(int layers, int heads, int head_dim, int max_text, rtr_dtype dt, int device,
                                rtr_xattn **out) {
    if (!out) return RTR_E_INVAL;
    *out = nullptr;
    if (layers < 1 || !shape_ok(heads, head_dim) || max_text < 1 || max_text > (1 << 24) ||
        (dt != RTR_BF16 && dt != RTR_F32) || device < 0)
        return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    rtr_xattn *x = new (std::nothrow) rtr_xattn();
    if (!x) return RTR_E_NOMEM;
    x->layers = layers; x->heads = heads; x->head_dim = head_dim; x->max_text = max_text;
    x->dt = dt; x->device = device;
    x->layer_bytes = (size_t)heads * max_text * head_dim * elt_size(dt);
    const size_t total = x->layer_bytes * layers;
    x->kbuf = guarded_alloc(total);
    x->vbuf = x->kbuf ? guarded_alloc(total) : nullptr;
    if (!x->kbuf || !x->vbuf) {
        guarded_free(x->kbuf);
        delete x;
        return RTR_E_NOMEM;
    }
    if (cudaMemset(x->kbuf, 0, total) != cudaSuccess || cudaMemset(x->vbuf, 0, total) != cudaSuccess) {
        guarded_free(x->kbuf); guarded_free(x->vbuf); delete x;
        return RTR_E_CUDA;
    }
    x->n_text.assign(layers, 0);
    if (dt == RTR_BF16) {
        x->tmk.resize(layers);
        x->tmv.resize(layers);
        x->tmk64.resize(layers);
        for (int l = 0; l < layers; ++l) {
            if (!make_tmap_bf16(&x->tmk[l], x->kbuf + l * x->layer_bytes, head_dim, max_text, heads, 128, 1) ||
                !make_tmap_bf16(&x->tmk64[l], x->kbuf + l * x->layer_bytes, head_dim, max_text, heads, 64, 1) ||
                !make_tmap_bf16(&x->tmv[l], x->vbuf + l * x->layer_bytes, head_dim, max_text, heads, 128, 1)) {
                guarded_free(x->kbuf); guarded_free(x->vbuf); delete x;
                return RTR_E_CUDA;
            }
        }
    }
    if (cudaDeviceSynchronize() != cudaSuccess) {
        guarded_free(x->kbuf); guarded_free(x->vbuf); delete x;
        return RTR_E_CUDA;
    }
    *out = x;
    return RTR_OK;
}

void rtr_crossattn_destroy(rtr_xattn *x) {
    if (!x) return;
    DeviceGuard dg(x->device);
    cudaDeviceSynchronize();
    guarded_free(x->kbuf);
    guarded_free(x->vbuf);
    delete x;
}

rtr_status rtr_crossattn_set_text(rtr_xattn *x, int layer, const void *k_text, const void *v_text, int n_text,
                                  rtr_stream_t stream) {
    if (!x || layer < 0 || layer >= x->layers || !aligned16(k_text) || !aligned16(v_text)) return RTR_E_INVAL;
    if (n_text < 1 || n_text > x->max_text) return RTR_E_INVAL;
    DeviceGuard dg(x->device);
    ScatterArgs a;
    a.src_k = k_text; a.src_v = v_text;
    a.dst_k = x->kbuf + layer * x->layer_bytes;
    a.dst_v = x->vbuf + layer * x->layer_bytes;
    a.n_tok = n_text; a.heads = x->heads; a.row_bytes = x->head_dim * (int)elt_size(x->dt);
    a.k_frame = n_text; a.first_slot = 0; a.slot_mod = 1; a.slot_off = 0;
    a.rows_per_head = x->max_text;
    rtr_status st = cuda_status(launch_kv_scatter(a, (cudaStream_t)stream));
    if (st == RTR_OK) x->n_text[layer] = n_text;
    return st;
}

rtr_status rtr_crossattn_reset(rtr_xattn *x) {
    if (!x) return RTR_E_INVAL;
    std::fill(x->n_text.begin(), x->n_text.end(), 0);
    return RTR_OK;
}

rtr_status rtr_crossattn_check_guards(const rtr_xattn *x) {
    if (!x) return RTR_E_INVAL;
    DeviceGuard dg(x->device);
    const size_t total = x->layer_bytes * x->layers;
    const rtr_status a = guards_status(x->kbuf, total);
    return a != RTR_OK ? a : guards_status(x->vbuf, total);
}

rtr_status rtr_test_fail_allocs(int after, int n) {
    if (after < 0 || n < 0) return RTR_E_INVAL;
    std::lock_guard<std::mutex> lock(g_alloc_mu);
    g_alloc_skip = after;
    g_alloc_fail = n;
    return RTR_OK;
}

rtr_status rtr_attn_cross(const rtr_xattn *x, int layer, const void *q, int n_q, void *out, float scale,
                          rtr_stream_t stream) {
    if (!x || layer < 0 || layer >= x->layers || n_q < 0) return RTR_E_INVAL;
    if (x->n_text[layer] == 0) return RTR_E_STATE;
    if (n_q == 0) return RTR_OK;
    if (!aligned16(q) || !aligned16(out)) return RTR_E_INVAL;
    AttnProblem pb;
    memset(&pb, 0, sizeof(pb));
    pb.nq = n_q; pb.heads = x->heads; pb.head_dim = x->head_dim; pb.kpf = 1;
    pb.nseg = 1;
    pb.seg[0] = KvSeg{0, 0, x->n_text[layer], 0};
    pb.scale = resolve_scale(scale, x->head_dim);
    pb.q = q; pb.o = out;
    pb.k0 = x->kbuf + layer * x->layer_bytes; pb.v0 = x->vbuf + layer * x->layer_bytes; pb.rows0 = x->max_text;
    DeviceGuard dg(x->device);
    const CUtensorMap *tk = x->dt == RTR_BF16 ? &x->tmk[layer] : nullptr;
    const CUtensorMap *tkh = x->dt == RTR_BF16 ? &x->tmk64[layer] : nullptr;
    const CUtensorMap *tv = x->dt == RTR_BF16 ? &x->tmv[layer] : nullptr;
    return run_attention(pb, x->dt, tk, tkh, tv, x->device, (cudaStream_t)stream);
}

unsigned long long rtr_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

rtr_status rtr_release_workspaces(int device, int *held_before) {
    if (device < 0) return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    if (held_before) *held_before = (int)workspace_count(device);
    return release_workspaces(device);
}

rtr_status rtr_test_inject_wait_timeout(int device, int launches) {
    if (device < 0 || device >= 64 || launches < 0) return RTR_E_INVAL;
    inject_wait_timeouts(device, launches);
    return RTR_OK;
}

rtr_status rtr_get_device_status(int device, rtr_stream_t stream) {
    if (device < 0) return RTR_E_INVAL;
    DeviceGuard dg(device);
    if (!dg.ok) return RTR_E_INVAL;
    unsigned *p = device_status_ptr(device);
    if (!p) return RTR_E_CUDA;
    unsigned h = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RTR_E_CUDA;
    if (cudaMemcpy(&h, p, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return RTR_E_CUDA;
    const unsigned zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return RTR_E_CUDA;
    return h == 0 ? RTR_OK : (rtr_status)h;
}

}  // extern "C"
