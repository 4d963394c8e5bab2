// topk.cu -- a3: exact top-k of fp32 scores per sequence (ties to the lower
// candidate index), reported as ascending positions.
// (arXiv 2606.09079: the Lightning Indexer's fine top-k inside the kept set,
// gist.science explainer 2.1 "Gestufte Selektion", cjcn.com.cn article section 2.)
//
// One CTA of 1024 threads per sequence.  A 4-pass, 8-bit radix select over
// order-preserving uint32 keys finds the k-th largest key T and how many of
// the keys equal to T are taken; an order-preserving block scan then emits
// every candidate with key > T and the first `need` candidates with key == T,
// in candidate order, which is ascending position.
#include "block_scan.cuh"
#include "common.cuh"

namespace lsa {

constexpr int kTopkThreads = 1024;

int launch_li_scores(const uint16_t *, const uint16_t *, const uint16_t *, int64_t, const int32_t *, int,
                     const int32_t *, const int32_t *, int, const int32_t *, const int32_t *, int, int, int, float *,
                     int32_t *, cudaStream_t);
bool indexer_shape_ok(int H, int D);

struct CandFromKept {   // candidate j -> token position kept[j / 64] * 64 + j % 64
    const int32_t *kept;
    __device__ int operator()(int j) const { return kept[j >> 6] * LSA_CHUNK + (j & 63); }
};
struct CandIdentity {
    __device__ int operator()(int j) const { return j; }
};

// grid B: cold[b] = number of kept chunks of sequence b that lie before its
// recent window (they contribute the top-k candidates).  One coalesced pass
// over the kept list, so the kernels that follow read a single count.
__global__ void __launch_bounds__(256) cold_count_kernel(const int32_t *__restrict__ kept_idx,
                                                         const int32_t *__restrict__ kept_count, int kept_cap,
                                                         const int32_t *__restrict__ window_start,
                                                         int32_t *__restrict__ cold) {
    __shared__ int part[8];
    const int b = blockIdx.x;
    const int cnt = min(max(kept_count[b], 0), kept_cap);
    const int fw = window_start[b] / LSA_CHUNK;
    const int32_t *kept = kept_idx + (size_t)b * kept_cap;
    int c = 0;
    for (int i = threadIdx.x; i < cnt; i += 256) c += kept[i] < fw;
    c = __reduce_add_sync(0xffffffffu, c);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < 8; ++w) t += part[w];
        cold[b] = t;
    }
}

// Adds 1 to hist[bin] for every lane with `active`, one shared atomic per distinct bin.
__device__ __forceinline__ void warp_hist_add(int *hist, uint32_t bin, bool active) {
    const unsigned act = __ballot_sync(0xffffffffu, active);
    if (!active) return;
    const unsigned same = __match_any_sync(act, bin);
    if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
}

// Scores of one sequence: from shared memory when they were staged there, else global.
template <class PosFn>
__device__ void topk_block(const float *__restrict__ s_glob, const float *s, int n, int k, PosFn pos,
                           int32_t *__restrict__ out, int32_t *__restrict__ out_count) {
    __shared__ int hist[256];
    __shared__ int warp_tot[kTopkThreads / 32 + 1];
    __shared__ uint32_t sh_prefix;
    __shared__ int sh_remaining;
    const int t = threadIdx.x;
    (void)s_glob;

    if (n <= k) {  // everything is selected, already in ascending order
        for (int j = t; j < k; j += kTopkThreads) out[j] = j < n ? pos(j) : -1;
        if (t == 0) *out_count = n;
        return;
    }

    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
    const int n_round = (n + kTopkThreads - 1) / kTopkThreads * kTopkThreads;   // warp-uniform trip count
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        if (t < 256) hist[t] = 0;
        __syncthreads();
        for (int j = t; j < n_round; j += kTopkThreads) {
            const uint32_t u = j < n ? ordered_key(s[j]) : 0u;
            warp_hist_add(hist, (u >> shift) & 255u, j < n && (u & pmask) == prefix);
        }
        __syncthreads();
        // suffix counts over digits, highest digit first
        int v = t < 256 ? hist[255 - t] : 0;
        int total;
        int excl = block_exclusive_scan<kTopkThreads>(v, warp_tot, &total);
        if (t < 256) {
            int incl = excl + v;
            if (incl >= remaining && excl < remaining) {
                sh_prefix = prefix | (uint32_t(255 - t) << shift);
                sh_remaining = remaining - excl;
            }
        }
        __syncthreads();
        prefix = sh_prefix;
        remaining = sh_remaining;
        pmask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;
    const int need_eq = remaining;  // keys equal to T that are taken, >= 1

    const int seg = (n + kTopkThreads - 1) / kTopkThreads;
    const int j0 = min(n, t * seg), j1 = min(n, j0 + seg);
    int gt = 0, eq = 0;
    for (int j = j0; j < j1; ++j) {
        uint32_t u = ordered_key(s[j]);
        gt += u > T;
        eq += u == T;
    }
    int dummy;
    int eq_before = block_exclusive_scan<kTopkThreads>(eq, warp_tot, &dummy);
    int take_eq = min(eq, max(0, need_eq - eq_before));
    int o = block_exclusive_scan<kTopkThreads>(gt + take_eq, warp_tot, &dummy);
    for (int j = j0; j < j1; ++j) {
        uint32_t u = ordered_key(s[j]);
        if (u > T || (u == T && take_eq > 0)) {
            if (u == T) --take_eq;
            out[o++] = pos(j);
        }
    }
    if (t == 0) *out_count = k;
}

// Copies n scores into dynamic shared memory when they fit; returns the array to read.
__device__ __forceinline__ const float *stage_scores(const float *__restrict__ g, int n, int cap) {
    extern __shared__ float stage[];
    if (n > cap) return g;
    const int n4 = (reinterpret_cast<uintptr_t>(g) & 15) == 0 ? n / 4 : 0;
    for (int i = threadIdx.x; i < n4; i += kTopkThreads)
        reinterpret_cast<float4 *>(stage)[i] = reinterpret_cast<const float4 *>(g)[i];
    for (int i = 4 * n4 + threadIdx.x; i < n; i += kTopkThreads) stage[i] = g[i];
    __syncthreads();
    return stage;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kept_kernel(const float *__restrict__ scores, int kept_cap,
                                                                 const int32_t *__restrict__ kept_idx,
                                                                 const int32_t *__restrict__ cold, int k,
                                                                 int32_t *__restrict__ topk_idx,
                                                                 int32_t *__restrict__ topk_count, int stage_cap) {
    const int b = blockIdx.x;
    const int32_t *kept = kept_idx + (size_t)b * kept_cap;
    const int n = cold[b] * LSA_CHUNK;
    const float *g = scores + (size_t)b * kept_cap * LSA_CHUNK;
    const float *s = n > k ? stage_scores(g, n, stage_cap) : g;
    topk_block(g, s, n, k, CandFromKept{kept}, topk_idx + (size_t)b * k, topk_count + b);
}

__global__ void __launch_bounds__(kTopkThreads) topk_scores_kernel(const float *__restrict__ scores,
                                                                   const int64_t *__restrict__ off, int max_cand,
                                                                   int k, int32_t *__restrict__ topk_idx,
                                                                   int32_t *__restrict__ topk_count, int stage_cap) {
    const int b = blockIdx.x;
    const int64_t a = off[b];
    const int n = (int)max((int64_t)0, min(off[b + 1] - a, (int64_t)max_cand));
    const float *s = n > k ? stage_scores(scores + a, n, stage_cap) : scores + a;
    topk_block(scores + a, s, n, k, CandIdentity{}, topk_idx + (size_t)b * k, topk_count + b);
}

// Scores staged in shared memory: up to 200 KB (51,200 candidates), never more than needed.
static int stage_capacity(int max_n) { return max(0, min(max_n, 51200)); }

}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_topk_workspace_size(int B, int kept_cap) {
    if (B <= 0 || kept_cap <= 0) return 0;
    Carver c(nullptr);
    c.take<int32_t>((size_t)B);                                   // kept cold chunk count per sequence
    c.take<float>((size_t)B * kept_cap * LSA_CHUNK);             // candidate scores (unless the caller passes them)
    return align_up(c.used, 256);
}

extern "C" int lsa_topk(const lsa_bf16 *q_li, const lsa_bf16 *w_li, const lsa_bf16 *li_pool, int64_t n_slots,
                        const int32_t *chunk_table, int table_stride, const int32_t *kept_idx,
                        const int32_t *kept_count, int kept_cap, const int32_t *window_start, int B, int Hl, int dl,
                        int k, int32_t *topk_idx, int32_t *topk_count, float *scores, int32_t *dev_status, void *ws,
                        size_t ws_bytes, lsa_stream_t stream) {
    LSA_REQUIRE(B > 0 && kept_cap > 0 && table_stride > 0 && n_slots > 0, LSA_ERR_INVALID_ARG,
                "lsa_topk: bad sizes (B=%d kept_cap=%d table_stride=%d n_slots=%lld)", B, kept_cap, table_stride,
                (long long)n_slots);
    LSA_REQUIRE(q_li && w_li && li_pool && chunk_table && kept_idx && kept_count && window_start && topk_idx &&
                    topk_count,
                LSA_ERR_INVALID_ARG, "lsa_topk: null pointer");
    LSA_REQUIRE(indexer_shape_ok(Hl, dl), LSA_ERR_SHAPE,
                "lsa_topk: unsupported Hl=%d dl=%d (dl in {64,128}, Hl multiple of 8 up to 128)", Hl, dl);
    LSA_REQUIRE(k >= 1 && k <= 65536, LSA_ERR_INVALID_ARG, "lsa_topk: k=%d outside [1, 65536]", k);
    LSA_REQUIRE((int64_t)kept_cap * LSA_CHUNK < (int64_t)1 << 31, LSA_ERR_INVALID_ARG, "lsa_topk: kept_cap too large");
    LSA_REQUIRE(ws && ws_bytes >= lsa_topk_workspace_size(B, kept_cap), LSA_ERR_WORKSPACE,
                "lsa_topk: workspace of %zu bytes, %zu needed", ws_bytes, lsa_topk_workspace_size(B, kept_cap));
    Carver c(ws);
    int32_t *cold = c.take<int32_t>((size_t)B);
    float *buf = c.take<float>((size_t)B * kept_cap * LSA_CHUNK);
    if (scores) buf = scores;
    cold_count_kernel<<<B, 256, 0, stream>>>(kept_idx, kept_count, kept_cap, window_start, cold);
    int rc = check_launch("cold_count_kernel");
    if (rc) return rc;
    rc = launch_li_scores(q_li, w_li, li_pool, n_slots, chunk_table, table_stride, kept_idx, kept_count, kept_cap,
                          window_start, cold, B, Hl, dl, buf, dev_status, stream);
    if (rc) return rc;
    const int cap = stage_capacity(kept_cap * LSA_CHUNK);
    LSA_CUDA(cudaFuncSetAttribute(topk_kept_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(cap * sizeof(float))));
    topk_kept_kernel<<<B, kTopkThreads, cap * sizeof(float), stream>>>(buf, kept_cap, kept_idx, cold, k, topk_idx,
                                                                       topk_count, cap);
    return check_launch("topk_kept_kernel");
}

extern "C" int lsa_topk_from_scores(const float *scores, const int64_t *cand_offset, int B, int max_cand, int k,
                                    int32_t *topk_idx, int32_t *topk_count, void *ws, size_t ws_bytes,
                                    lsa_stream_t stream) {
    (void)ws; (void)ws_bytes;
    LSA_REQUIRE(B > 0 && scores && cand_offset && topk_idx && topk_count, LSA_ERR_INVALID_ARG,
                "lsa_topk_from_scores: null pointer or B <= 0");
    LSA_REQUIRE(max_cand >= 0, LSA_ERR_INVALID_ARG, "lsa_topk_from_scores: max_cand must be >= 0");
    LSA_REQUIRE(k >= 1 && k <= 65536, LSA_ERR_INVALID_ARG, "lsa_topk_from_scores: k=%d outside [1, 65536]", k);
    const int cap = stage_capacity(max_cand);
    LSA_CUDA(cudaFuncSetAttribute(topk_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(cap * sizeof(float))));
    topk_scores_kernel<<<B, kTopkThreads, cap * sizeof(float), stream>>>(scores, cand_offset, max_cand, k, topk_idx,
                                                                         topk_count, cap);
    return check_launch("topk_scores_kernel");
}
