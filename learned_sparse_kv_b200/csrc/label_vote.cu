// label_vote.cu -- a7 (offline): cross-layer majority-vote labels for one window.
// (arXiv 2606.09079: softmax, nucleus top-p 0.6, at least 3 layers; gist.science
// explainer 2.2, cjcn.com.cn article section 3.)
//
// Kernel 1, one CTA per (layer, step): softmax normaliser, bitonic sort of
// (score desc, index asc) in shared memory, block prefix sum of exp(s - max) in
// sorted order, nucleus cut at the first prefix reaching top_p * Z, and an
// atomicOr of the layer's bit into mask[step][chunk].  Kernel 2, per chunk:
// per-step popcounts -> votes and labels.
#include <mutex>

#include "common.cuh"
#include "nvtx_range.cuh"

namespace lsa {

constexpr int kVoteThreads = 1024;
constexpr int kMaxVoteChunks = 16384;

__device__ __forceinline__ bool before(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

__device__ float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) red[wid] = v;
    __syncthreads();
    float t = 0.f;
    if (wid == 0) {
        t = lane < kVoteThreads / 32 ? red[lane] : 0.f;
        t = warp_sum(t);
        if (lane == 0) red[32] = t;
    }
    __syncthreads();
    t = red[32];
    __syncthreads();
    return t;
}

__device__ float block_max(float v, float *red) {
    v = warp_max(v);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) red[wid] = v;
    __syncthreads();
    float t = -INFINITY;
    if (wid == 0) {
        t = lane < kVoteThreads / 32 ? red[lane] : -INFINITY;
        t = warp_max(t);
        if (lane == 0) red[32] = t;
    }
    __syncthreads();
    t = red[32];
    __syncthreads();
    return t;
}

// Exclusive scan of one float per thread (block of kVoteThreads).
__device__ float block_exclusive_scan_f(float v, float *red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    float inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) red[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        float t = red[lane];
        float ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float n = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += n;
        }
        red[lane] = ti - t;
    }
    __syncthreads();
    float res = red[wid] + inc - v;
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kVoteThreads) nucleus_mark_kernel(const float *__restrict__ scores, int n_layers,
                                                                    int n_steps, int n, int npow2, float top_p,
                                                                    uint32_t *__restrict__ masks, int words) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *key = reinterpret_cast<float *>(smem_raw);
    int *idx = reinterpret_cast<int *>(key + npow2);
    __shared__ float red[33];
    __shared__ int first_hit;
    const int l = blockIdx.x / n_steps, t = blockIdx.x % n_steps;
    const float *s = scores + ((size_t)l * n_steps + t) * n;
    const int tid = threadIdx.x;

    float mx = -INFINITY;
    for (int i = tid; i < npow2; i += kVoteThreads) {
        float v = i < n ? s[i] : -INFINITY;
        key[i] = v;
        idx[i] = i;
        mx = fmaxf(mx, v);
    }
    if (tid == 0) first_hit = n;
    const float m = block_max(mx, red);
    float z = 0.f;
    for (int i = tid; i < n; i += kVoteThreads) z += expf(key[i] - m);
    const float Z = block_sum(z, red);

    // bitonic sort into (score desc, index asc); padding (-inf, index >= n) sorts last
    for (int size = 2; size <= npow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = tid; i < npow2 / 2; i += kVoteThreads) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;  // this run is ordered "before" first
                float ka = key[lo], kb = key[hi];
                int ia = idx[lo], ib = idx[hi];
                if (before(kb, ib, ka, ia) == up) {
                    key[lo] = kb; key[hi] = ka;
                    idx[lo] = ib; idx[hi] = ia;
                }
            }
        }
    }
    __syncthreads();

    // prefix sums of exp(s - m) in sorted order; first position reaching top_p * Z
    const int seg = (n + kVoteThreads - 1) / kVoteThreads;
    const int i0 = min(n, tid * seg), i1 = min(n, i0 + seg);
    float local = 0.f;
    for (int i = i0; i < i1; ++i) local += expf(key[i] - m);
    float run = block_exclusive_scan_f(local, red);
    const float thr = top_p * Z;
    for (int i = i0; i < i1; ++i) {
        run += expf(key[i] - m);
        if (run >= thr) {
            atomicMin(&first_hit, i);
            break;
        }
    }
    __syncthreads();
    const int taken = min(n, first_hit + 1);
    const uint32_t bit = 1u << (l & 31);
    for (int i = tid; i < taken; i += kVoteThreads)
        if (idx[i] < n) atomicOr(&masks[((size_t)t * n + idx[i]) * words + (l >> 5)], bit);
}

__global__ void vote_kernel(const uint32_t *__restrict__ masks, int n_steps, int n, int words, int min_layers,
                            int mode, uint8_t *__restrict__ labels, int32_t *__restrict__ max_votes) {
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < n; c += gridDim.x * blockDim.x) {
        int best = 0;
        uint32_t any0 = 0, any1 = 0;
        for (int t = 0; t < n_steps; ++t) {
            const uint32_t *m = masks + ((size_t)t * n + c) * words;
            uint32_t w0 = m[0], w1 = words > 1 ? m[1] : 0u;
            best = max(best, __popc(w0) + __popc(w1));
            any0 |= w0;
            any1 |= w1;
        }
        if (mode == 1) best = __popc(any0) + __popc(any1);
        labels[c] = best >= min_layers;
        if (max_votes) max_votes[c] = best;
    }
}

}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_label_vote_workspace_size(int n_layers, int n_steps, int n_chunks) {
    if (n_layers <= 0 || n_steps <= 0 || n_chunks <= 0) return 0;
    const int words = (n_layers + 31) / 32;
    return align_up((size_t)n_steps * n_chunks * words * sizeof(uint32_t), 256);
}

extern "C" int lsa_label_vote(const float *scores, int n_layers, int n_steps, int n_chunks, float top_p,
                              int min_layers, int mode, uint8_t *labels, int32_t *max_votes, void *ws,
                              size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(scores && labels, LSA_ERR_INVALID_ARG, "lsa_label_vote: null pointer");
    LSA_REQUIRE(n_layers >= 1 && n_layers <= 64 && n_steps >= 1 && n_chunks >= 1 && n_chunks <= kMaxVoteChunks,
                LSA_ERR_SHAPE, "lsa_label_vote: unsupported sizes (layers=%d steps=%d chunks=%d)", n_layers, n_steps,
                n_chunks);
    LSA_REQUIRE(mode == 0 || mode == 1, LSA_ERR_INVALID_ARG, "lsa_label_vote: mode must be 0 or 1");
    LSA_REQUIRE(top_p > 0.f, LSA_ERR_INVALID_ARG, "lsa_label_vote: top_p must be positive");
    const size_t need = lsa_label_vote_workspace_size(n_layers, n_steps, n_chunks);
    LSA_REQUIRE(ws && ws_bytes >= need, LSA_ERR_WORKSPACE, "lsa_label_vote: workspace of %zu bytes, %zu needed",
                ws_bytes, need);
    const int words = (n_layers + 31) / 32;
    uint32_t *masks = static_cast<uint32_t *>(ws);
    LSA_CUDA(cudaMemsetAsync(masks, 0, (size_t)n_steps * n_chunks * words * sizeof(uint32_t), stream));
    int npow2 = 2;
    while (npow2 < n_chunks) npow2 <<= 1;
    const size_t smem = (size_t)npow2 * (sizeof(float) + sizeof(int));
    LSA_CUDA(cudaFuncSetAttribute(nucleus_mark_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    nucleus_mark_kernel<<<n_layers * n_steps, kVoteThreads, smem, stream>>>(scores, n_layers, n_steps, n_chunks, npow2,
                                                                            top_p, masks, words);
    int rc = check_launch("nucleus_mark_kernel");
    if (rc) return rc;
    vote_kernel<<<(n_chunks + 255) / 256, 256, 0, stream>>>(masks, n_steps, n_chunks, words, min_layers, mode, labels,
                                                            max_votes);
    return check_launch("vote_kernel");
}

// ----------------------------------------------------------------------------
// Label vote for callers that cannot allocate device memory.
//
// The vote needs one word per (step, chunk) of scratch.  Callers that may not
// allocate -- code that runs where the device allocator must not be entered,
// or a host that budgets every device byte up front and hands this library
// only its inputs and outputs -- get that scratch from the fixed array below,
// which every GPU that loads the library holds until the process exits.
namespace lsa {

constexpr size_t kStaticVoteWords = size_t(1) << 20;   // 4 MiB of uint32 vote masks
static __device__ __align__(256) uint32_t g_vote_scratch[kStaticVoteWords];

static std::mutex g_vote_scratch_lock;
static uint32_t *g_vote_scratch_dev[64];   // device address of g_vote_scratch, per device

// Host code may not use g_vote_scratch itself (it names a host-side stand-in);
// the device address is looked up once per device, with that device current.
// The cached address belongs to the device's context at that time: after a
// cudaDeviceReset of the device it is stale, and this entry point must not be
// called on that device again in the same process.
static int vote_scratch(uint32_t **out) {
    int dev = 0;
    LSA_CUDA(cudaGetDevice(&dev));
    LSA_REQUIRE(dev >= 0 && dev < 64, LSA_ERR_INVALID_ARG, "lsa_label_vote_noalloc: device %d out of range", dev);
    std::lock_guard<std::mutex> guard(g_vote_scratch_lock);
    if (!g_vote_scratch_dev[dev]) {
        void *p = nullptr;
        LSA_CUDA(cudaGetSymbolAddress(&p, g_vote_scratch));
        g_vote_scratch_dev[dev] = static_cast<uint32_t *>(p);
    }
    *out = g_vote_scratch_dev[dev];
    return LSA_OK;
}

}  // namespace lsa

extern "C" int lsa_label_vote_noalloc(const float *scores, int n_layers, int n_steps, int n_chunks, float top_p,
                                      int min_layers, int mode, uint8_t *labels, int32_t *max_votes,
                                      lsa_stream_t stream) {
    LSA_REQUIRE(scores && labels, LSA_ERR_INVALID_ARG, "lsa_label_vote_noalloc: null pointer");
    LSA_REQUIRE(n_layers >= 1 && n_layers <= 64 && n_steps >= 1 && n_chunks >= 1 && n_chunks <= kMaxVoteChunks,
                LSA_ERR_SHAPE, "lsa_label_vote_noalloc: unsupported sizes (layers=%d steps=%d chunks=%d)", n_layers,
                n_steps, n_chunks);
    LSA_REQUIRE(mode == 0 || mode == 1, LSA_ERR_INVALID_ARG, "lsa_label_vote_noalloc: mode must be 0 or 1");
    LSA_REQUIRE(top_p > 0.f, LSA_ERR_INVALID_ARG, "lsa_label_vote_noalloc: top_p must be positive");
    const int words = (n_layers + 31) / 32;
    const size_t need = (size_t)n_steps * n_chunks * words;
    LSA_REQUIRE(need <= kStaticVoteWords, LSA_ERR_CAPACITY,
                "lsa_label_vote_noalloc: steps x chunks x ceil(layers/32) = %zu exceeds the built-in scratch of %zu "
                "words; use lsa_label_vote with a caller workspace",
                need, kStaticVoteWords);
    uint32_t *masks = nullptr;
    int rc = vote_scratch(&masks);
    if (rc) return rc;
    LSA_CUDA(cudaMemsetAsync(masks, 0, need * sizeof(uint32_t), stream));   // every call starts from zero
    int npow2 = 2;
    while (npow2 < n_chunks) npow2 <<= 1;
    const size_t smem = (size_t)npow2 * (sizeof(float) + sizeof(int));
    LSA_CUDA(cudaFuncSetAttribute(nucleus_mark_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    nucleus_mark_kernel<<<n_layers * n_steps, kVoteThreads, smem, stream>>>(scores, n_layers, n_steps, n_chunks, npow2,
                                                                            top_p, masks, words);
    rc = check_launch("nucleus_mark_kernel");
    if (rc) return rc;
    vote_kernel<<<(n_chunks + 255) / 256, 256, 0, stream>>>(masks, n_steps, n_chunks, words, min_layers, mode, labels,
                                                            max_votes);
    return check_launch("vote_kernel");
}
