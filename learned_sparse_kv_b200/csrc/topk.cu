// topk.cu -- a3: exact top-k of fp32 scores per sequence (ties to the lower
// candidate index), reported as ascending positions.
// (arXiv 2606.09079: the Lightning Indexer's fine top-k inside the kept set,
// gist.science explainer 2.1 "Gestufte Selektion", cjcn.com.cn article section 2.)
//
// One cluster of 8 CTAs per sequence.  A 4-pass, 8-bit radix select over
// order-preserving uint32 keys finds the k-th largest key T and how many of
// the keys equal to T are taken; an order-preserving scan over the cluster then
// emits every candidate with key > T and the first `need` candidates with
// key == T, in candidate order, which is ascending position.
#include "block_scan.cuh"
#include "common.cuh"
#include "nvtx_range.cuh"
#include "sm100.cuh"

namespace lsa {

constexpr int kTopkThreads = 512;   // threads per CTA
// CTAs per sequence: one thread-block cluster.  8 measured fastest of 1..16 for 8 sequences of
// ~16K candidates; a single sequence (a batch of one) takes 16, so that twice the multiprocessors
// share its candidates.
constexpr int kTopkCtas = 8, kTopkCtasOne = 16;

int launch_li_scores(const uint16_t *, const uint16_t *, const uint16_t *, int64_t, const int32_t *, int,
                     const int32_t *, const int32_t *, int, const int32_t *, int32_t *, int, int, int, float *,
                     int32_t *, cudaStream_t, const AppendArgs *);
bool indexer_shape_ok(int H, int D);
bool indexer_counts_cold(int H, int D, int B);

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

// Adds 1 to hist[bin] for every lane with `active`.  Plain shared atomics:
// aggregating equal bins across the warp first (match.any) measured slower.
__device__ __forceinline__ void warp_hist_add(int *hist, uint32_t bin, bool active) {
    if (active) atomicAdd(&hist[bin], 1);
}

__device__ __forceinline__ int ld_cluster_s32(const void *p, uint32_t rank) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];\n" : "=r"(v) : "r"(sm100::map_to_rank(p, rank)) : "memory");
    return v;
}

struct TopkShared {
    int hist[2][256];                     // digit counts of this CTA's slice, double-buffered by pass
    int warp_tot[kTopkThreads / 32 + 1];
    int cnt[2];                           // this CTA's counts of keys > T and == T
    int base, eq_lower;                   // output offset of this CTA, keys == T in lower CTAs
    uint32_t prefix;
    int remaining, in_bin;
};

// Top-k of the n scores of one sequence by the NC CTAs of a cluster.
// CTA c takes the contiguous slice [c seg, (c + 1) seg) and stages its keys in
// shared memory when they fit (stage_cap keys).  Each 8-bit radix pass counts
// digits locally; after a cluster barrier every CTA sums the NC
// histograms through distributed shared memory and picks the same digit, so
// no result has to be broadcast.  The passes stop as soon as the chosen digit's
// bin holds exactly the keys still to be taken (then every key of the bin is
// selected and its lower digits do not matter).  The emission is ordered: a
// CTA's output offset is the number of selected keys in the lower slices, and
// ties at the threshold go to the lowest candidate indices.
template <int NC, class PosFn>
__device__ void topk_cluster(const float *__restrict__ s, int n, int k, PosFn pos, int32_t *__restrict__ out,
                             int32_t *__restrict__ out_count, int stage_cap) {
    __shared__ TopkShared sh;
    extern __shared__ uint32_t keys[];
    const int t = threadIdx.x;
    const int c = (int)sm100::cluster_rank();

    if (n <= k) {  // everything is selected, already in ascending order
        for (int j = c * kTopkThreads + t; j < k; j += NC * kTopkThreads) out[j] = j < n ? pos(j) : -1;
        if (c == 0 && t == 0) *out_count = n;
        return;
    }
    const int seg = (n + NC - 1) / NC;
    const int j0 = min(n, c * seg), len = min(n, j0 + seg) - j0;
    const bool staged = len <= stage_cap;
    if (staged)
        for (int i = t; i < len; i += kTopkThreads) keys[i] = ordered_key(s[j0 + i]);
    auto key = [&](int i) { return staged ? keys[i] : ordered_key(s[j0 + i]); };
    if (t < 256) {
        sh.hist[0][t] = 0;
        sh.hist[1][t] = 0;
    }
    __syncthreads();

    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
    const int len_round = (len + kTopkThreads - 1) / kTopkThreads * kTopkThreads;   // warp-uniform trip count
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        int *hist = sh.hist[pass & 1];   // zeroed, and ordered before these adds by a block barrier
        for (int i = t; i < len_round; i += kTopkThreads) {
            const uint32_t u = i < len ? key(i) : 0u;
            warp_hist_add(hist, (u >> shift) & 255u, i < len && (u & pmask) == prefix);
        }
        sm100::cluster_sync();   // every CTA's histogram of this pass is complete
        int v = 0;               // suffix counts over digits, highest digit first
        if (t < 256) {
            for (int r = 0; r < NC; ++r) v += ld_cluster_s32(&hist[255 - t], (uint32_t)r);
            // The other buffer serves the next pass: every CTA finished reading it
            // (in the previous pass) before the cluster barrier above.  Pass 1 finds
            // it zero from the start.
            if (pass >= 1 && pass < 3) sh.hist[(pass + 1) & 1][t] = 0;
        }
        int total;
        const int excl = block_exclusive_scan<kTopkThreads>(v, sh.warp_tot, &total);
        if (t < 256 && excl < remaining && excl + v >= remaining) {
            sh.prefix = prefix | (uint32_t(255 - t) << shift);
            sh.remaining = remaining - excl;
            sh.in_bin = v;
        }
        __syncthreads();
        prefix = sh.prefix;   // rewritten only after the next pass's barriers
        remaining = sh.remaining;
        pmask |= 255u << shift;
        if (sh.in_bin == remaining) break;   // the same in every CTA: all sum the same histograms
    }
    // Selected: keys whose digits so far exceed the threshold's, and the first need_eq
    // (in candidate order) of those equal to it.
    const uint32_t T = prefix;
    const int need_eq = remaining;  // keys equal to T that are taken, >= 1

    const int sub = (len + kTopkThreads - 1) / kTopkThreads;
    const int i0 = min(len, t * sub), i1 = min(len, i0 + sub);
    int gt = 0, eq = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = key(i) & pmask;
        gt += u > T;
        eq += u == T;
    }
    int gt_tot, eq_tot;
    const int eq_before = block_exclusive_scan<kTopkThreads>(eq, sh.warp_tot, &eq_tot);
    (void)block_exclusive_scan<kTopkThreads>(gt, sh.warp_tot, &gt_tot);
    if (t == 0) { sh.cnt[0] = gt_tot; sh.cnt[1] = eq_tot; }
    sm100::cluster_sync();   // every CTA's counts are published
    if (t < 32) {
        // Lane r < c reads CTA r's counts (all remote loads in flight at once); CTA r
        // contributes its keys above T and its share of the keys equal to T, which go
        // to the lowest CTAs first (eq_before_r = keys equal to T in CTAs below r).
        int g_r = 0, e_r = 0;
        if (t < c) {
            g_r = ld_cluster_s32(&sh.cnt[0], (uint32_t)t);
            e_r = ld_cluster_s32(&sh.cnt[1], (uint32_t)t);
        }
        int e_incl = e_r;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, e_incl, o);
            if (t >= o) e_incl += y;
        }
        const int eq_before_r = e_incl - e_r;
        const int base = __reduce_add_sync(0xffffffffu, g_r + min(e_r, max(0, need_eq - eq_before_r)));
        const int eq_lower = __reduce_add_sync(0xffffffffu, e_r);
        if (t == 0) {
            sh.base = base;
            sh.eq_lower = eq_lower;
        }
    }
    __syncthreads();
    int take_eq = min(eq, max(0, need_eq - (sh.eq_lower + eq_before)));
    int dummy;
    int o = sh.base + block_exclusive_scan<kTopkThreads>(gt + take_eq, sh.warp_tot, &dummy);
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = key(i) & pmask;
        if (u > T || (u == T && take_eq > 0)) {
            if (u == T) --take_eq;
            out[o++] = pos(j0 + i);
        }
    }
    if (c == 0 && t == 0) *out_count = k;
    sm100::cluster_sync();   // no CTA leaves while another may still read its counts
}

template <int NC>
__global__ void __launch_bounds__(kTopkThreads) topk_kept_kernel(const float *__restrict__ scores, int kept_cap,
                                                                 const int32_t *__restrict__ kept_idx,
                                                                 const int32_t *__restrict__ cold, int k,
                                                                 int32_t *__restrict__ topk_idx,
                                                                 int32_t *__restrict__ topk_count, int stage_cap) {
    const int b = blockIdx.y;
    const int32_t *kept = kept_idx + (size_t)b * kept_cap;
    const int n = min(max(cold[b], 0), kept_cap) * LSA_CHUNK;
    topk_cluster<NC>(scores + (size_t)b * kept_cap * LSA_CHUNK, n, k, CandFromKept{kept}, topk_idx + (size_t)b * k,
                 topk_count + b, stage_cap);
}

template <int NC>
__global__ void __launch_bounds__(kTopkThreads) topk_scores_kernel(const float *__restrict__ scores,
                                                                   const int64_t *__restrict__ off, int max_cand,
                                                                   int k, int32_t *__restrict__ topk_idx,
                                                                   int32_t *__restrict__ topk_count, int stage_cap) {
    const int b = blockIdx.y;
    const int64_t a = off[b];
    const int n = (int)max((int64_t)0, min(off[b + 1] - a, (int64_t)max_cand));
    topk_cluster<NC>(scores + a, n, k, CandIdentity{}, topk_idx + (size_t)b * k, topk_count + b, stage_cap);
}

// ------------------------------------------------------- baseline selectors --
// The pages compare LSA with a recency-only window and with random retention of
// a fraction of the older chunks (cjcn.com.cn article section 5, gist.science
// explainer section 4).  The random selector keeps, of the n_old chunks before
// the window, the m with the smallest SplitMix64 draws; as scores for the
// cluster top-k above they are 2^24 - 1 - draw, exact in fp32, so the m largest
// scores are the m smallest draws and ties go to the lower chunk index.

// Output number c of a SplitMix64 stream started at `seed` (Steele, Lea and
// Flood, OOPSLA 2014): state = seed + (c + 1) * golden-ratio increment, mixed.
__device__ __forceinline__ uint64_t splitmix64_output(uint64_t seed, uint64_t c) {
    uint64_t z = seed + (c + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ int older_chunks(const int32_t *window_start, int b, int max_old, int32_t *status) {
    const int n = max(window_start[b], 0) / LSA_CHUNK;
    if (n > max_old) {
        if (status && threadIdx.x == 0 && blockIdx.x == 0) flag(status, LSA_DEV_INDEX);
        return max_old;
    }
    return n;
}

// grid (ceil(max_old / 256), B): scores[b, s] for the older chunks s of sequence b.
__global__ void __launch_bounds__(256) random_score_kernel(const int32_t *__restrict__ window_start, int max_old,
                                                           uint64_t seed, float *__restrict__ scores) {
    const int b = blockIdx.y, s = blockIdx.x * 256 + threadIdx.x;
    const int n_old = min(max(window_start[b], 0) / LSA_CHUNK, max_old);
    if (s >= n_old) return;
    const uint32_t draw = (uint32_t)(splitmix64_output(seed, ((uint64_t)b << 32) + (uint64_t)s) >> 40);
    scores[(size_t)b * max_old + s] = (float)(0xFFFFFFu - draw);
}

// One cluster per sequence: the m = round(n_old * num / den) chunks with the largest
// scores, ascending, then -1 up to kept_cap.
template <int NC>
__global__ void __launch_bounds__(kTopkThreads) random_select_kernel(const float *__restrict__ scores,
                                                                     const int32_t *__restrict__ window_start,
                                                                     int max_old, int num, int den,
                                                                     int32_t *__restrict__ kept_idx,
                                                                     int32_t *__restrict__ kept_count, int kept_cap,
                                                                     int32_t *status, int stage_cap) {
    const int b = blockIdx.y;
    const int n_old = older_chunks(window_start, b, max_old, status);
    const int m = (int)min(((int64_t)n_old * num + den / 2) / den, (int64_t)n_old);   // <= kept_cap (host check)
    int32_t *out = kept_idx + (size_t)b * kept_cap;
    const int c = (int)sm100::cluster_rank();
    for (int j = m + c * kTopkThreads + (int)threadIdx.x; j < kept_cap; j += NC * kTopkThreads) out[j] = -1;
    if (m == 0) {
        if (c == 0 && threadIdx.x == 0) kept_count[b] = 0;
        return;
    }
    topk_cluster<NC>(scores + (size_t)b * max_old, n_old, m, CandIdentity{}, out, kept_count + b, stage_cap);
}

// Keys staged per CTA: a slice of at most ceil(max_n / 8), never more than 24,576 (96 KB).
static int cluster_ctas(int B) { return B == 1 ? kTopkCtasOne : kTopkCtas; }
static int stage_capacity(int max_n, int nc) { return max(0, min((max_n + nc - 1) / nc, 24576)); }

// One cluster of nc CTAs per sequence.
template <class... Args>
static int launch_topk(void (*kernel)(Args...), int nc, int B, int stage_cap, cudaStream_t stream, const char *what,
                       Args... args) {
    const size_t smem = (size_t)stage_cap * sizeof(uint32_t);
    LSA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    LSA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, B, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LSA_CUDA(cudaLaunchKernelEx(&cfg, kernel, args...));
    return check_launch(what);
}

}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_topk_workspace_size(int B, int kept_cap) {
    if (B <= 0 || kept_cap <= 0) return 0;
    Carver c(nullptr);
    c.take<int32_t>((size_t)B);                                   // kept cold chunk count per sequence
    c.take<float>((size_t)B * kept_cap * LSA_CHUNK);             // candidate scores (unless the caller passes them)
    return align_up(c.used, 256);
}

static int topk_impl(const lsa_bf16 *q_li, const lsa_bf16 *w_li, const lsa_bf16 *li_pool, int64_t n_slots,
                     const int32_t *chunk_table, int table_stride, const int32_t *kept_idx,
                     const int32_t *kept_count, int kept_cap, const int32_t *window_start, int B, int Hl, int dl,
                     int k, int32_t *topk_idx, int32_t *topk_count, float *scores, int32_t *dev_status, void *ws,
                     size_t ws_bytes, lsa_stream_t stream, const AppendArgs *app) {
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
    int rc = LSA_OK;
    if (!indexer_counts_cold(Hl, dl, B)) {
        cold_count_kernel<<<B, 256, 0, stream>>>(kept_idx, kept_count, kept_cap, window_start, cold);
        rc = check_launch("cold_count_kernel");
        if (rc) return rc;
    }
    rc = launch_li_scores(q_li, w_li, li_pool, n_slots, chunk_table, table_stride, kept_idx, kept_count, kept_cap,
                          window_start, cold, B, Hl, dl, buf, dev_status, stream, app);
    if (rc) return rc;
    const int nc = cluster_ctas(B), cap = stage_capacity(kept_cap * LSA_CHUNK, nc);
    if (nc == kTopkCtasOne)
        return launch_topk(topk_kept_kernel<kTopkCtasOne>, nc, B, cap, stream, "topk_kept_kernel",
                           (const float *)buf, kept_cap, kept_idx, (const int32_t *)cold, k, topk_idx, topk_count,
                           cap);
    return launch_topk(topk_kept_kernel<kTopkCtas>, nc, B, cap, stream, "topk_kept_kernel", (const float *)buf,
                       kept_cap, kept_idx, (const int32_t *)cold, k, topk_idx, topk_count, cap);
}

extern "C" int lsa_topk(const lsa_bf16 *q_li, const lsa_bf16 *w_li, const lsa_bf16 *li_pool, int64_t n_slots,
                        const int32_t *chunk_table, int table_stride, const int32_t *kept_idx,
                        const int32_t *kept_count, int kept_cap, const int32_t *window_start, int B, int Hl, int dl,
                        int k, int32_t *topk_idx, int32_t *topk_count, float *scores, int32_t *dev_status, void *ws,
                        size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    return topk_impl(q_li, w_li, li_pool, n_slots, chunk_table, table_stride, kept_idx, kept_count, kept_cap,
                     window_start, B, Hl, dl, k, topk_idx, topk_count, scores, dev_status, ws, ws_bytes, stream,
                     nullptr);
}

extern "C" int lsa_append_topk(const lsa_bf16 *new_kv, const lsa_bf16 *new_li, lsa_bf16 *kv_pool,
                               int64_t kv_row_stride, int kv_width, int32_t *window_len, const lsa_bf16 *q_li,
                               const lsa_bf16 *w_li, lsa_bf16 *li_pool, int64_t n_slots, const int32_t *chunk_table,
                               int table_stride, const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
                               const int32_t *window_start, int B, int Hl, int dl, int k, int32_t *topk_idx,
                               int32_t *topk_count, float *scores, int32_t *dev_status, void *ws, size_t ws_bytes,
                               lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(new_kv && new_li && kv_pool && window_len && li_pool, LSA_ERR_INVALID_ARG,
                "lsa_append_topk: null append pointer");
    LSA_REQUIRE(kv_width > 0 && kv_width % 8 == 0 && kv_row_stride >= kv_width && kv_row_stride % 8 == 0,
                LSA_ERR_INVALID_ARG, "lsa_append_topk: kv width/stride must be positive multiples of 8");
    auto al16 = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
    LSA_REQUIRE(al16(new_kv) && al16(new_li) && al16(kv_pool) && al16(li_pool), LSA_ERR_INVALID_ARG,
                "lsa_append_topk: rows are copied in 16-byte vectors: 16-byte aligned bases");
    if (!indexer_counts_cold(Hl, dl, B)) {
        // other indexer shapes: the append is a launch of its own, then the top-k call
        const int rc = lsa_append_token(new_kv, nullptr, new_li, kv_pool, kv_row_stride, kv_width, nullptr, 0, 0,
                                        li_pool, dl, n_slots, chunk_table, table_stride, window_start, window_len, B,
                                        dev_status, stream);
        if (rc) return rc;
        return lsa_topk(q_li, w_li, li_pool, n_slots, chunk_table, table_stride, kept_idx, kept_count, kept_cap,
                        window_start, B, Hl, dl, k, topk_idx, topk_count, scores, dev_status, ws, ws_bytes, stream);
    }
    const AppendArgs app = {new_kv, new_li, kv_pool, li_pool, kv_row_stride, kv_width, window_len};
    return topk_impl(q_li, w_li, li_pool, n_slots, chunk_table, table_stride, kept_idx, kept_count, kept_cap,
                     window_start, B, Hl, dl, k, topk_idx, topk_count, scores, dev_status, ws, ws_bytes, stream, &app);
}

extern "C" int lsa_topk_kernel_count(int B, int Hl, int dl) {
    if (B <= 0 || !indexer_shape_ok(Hl, dl)) return 0;
    return indexer_counts_cold(Hl, dl, B) ? 2 : 3;
}

extern "C" int lsa_topk_from_scores(const float *scores, const int64_t *cand_offset, int B, int max_cand, int k,
                                    int32_t *topk_idx, int32_t *topk_count, void *ws, size_t ws_bytes,
                                    lsa_stream_t stream) {
    LSA_ABI_RANGE();
    (void)ws; (void)ws_bytes;
    LSA_REQUIRE(B > 0 && scores && cand_offset && topk_idx && topk_count, LSA_ERR_INVALID_ARG,
                "lsa_topk_from_scores: null pointer or B <= 0");
    LSA_REQUIRE(max_cand >= 0, LSA_ERR_INVALID_ARG, "lsa_topk_from_scores: max_cand must be >= 0");
    LSA_REQUIRE(k >= 1 && k <= 65536, LSA_ERR_INVALID_ARG, "lsa_topk_from_scores: k=%d outside [1, 65536]", k);
    const int nc = cluster_ctas(B), cap = stage_capacity(max_cand, nc);
    if (nc == kTopkCtasOne)
        return launch_topk(topk_scores_kernel<kTopkCtasOne>, nc, B, cap, stream, "topk_scores_kernel", scores,
                           cand_offset, max_cand, k, topk_idx, topk_count, cap);
    return launch_topk(topk_scores_kernel<kTopkCtas>, nc, B, cap, stream, "topk_scores_kernel", scores, cand_offset,
                       max_cand, k, topk_idx, topk_count, cap);
}

extern "C" size_t lsa_select_baseline_workspace_size(int B, int max_old_chunks) {
    if (B <= 0 || max_old_chunks < 0) return 0;
    Carver c(nullptr);
    c.take<float>((size_t)B * (max_old_chunks > 0 ? max_old_chunks : 1));   // draws as top-k scores
    return align_up(c.used, 256);
}

extern "C" int lsa_select_baseline(int mode, const int32_t *window_start, int B, int max_old_chunks, uint64_t seed,
                                   int keep_num, int keep_den, int32_t *kept_idx, int32_t *kept_count, int kept_cap,
                                   int32_t *dev_status, void *ws, size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(mode == LSA_SELECT_RECENT || mode == LSA_SELECT_RANDOM, LSA_ERR_INVALID_ARG,
                "lsa_select_baseline: mode must be LSA_SELECT_RECENT or LSA_SELECT_RANDOM (got %d)", mode);
    LSA_REQUIRE(B > 0 && kept_cap >= 1 && max_old_chunks >= 0, LSA_ERR_INVALID_ARG,
                "lsa_select_baseline: bad sizes (B=%d kept_cap=%d max_old_chunks=%d)", B, kept_cap, max_old_chunks);
    LSA_REQUIRE(kept_idx && kept_count, LSA_ERR_INVALID_ARG, "lsa_select_baseline: null output pointer");
    if (mode == LSA_SELECT_RECENT) {
        LSA_CUDA(cudaMemsetAsync(kept_idx, 0xFF, sizeof(int32_t) * (size_t)B * kept_cap, stream));   // -1
        LSA_CUDA(cudaMemsetAsync(kept_count, 0, sizeof(int32_t) * (size_t)B, stream));
        return LSA_OK;
    }
    LSA_REQUIRE(window_start, LSA_ERR_INVALID_ARG, "lsa_select_baseline: null window_start");
    LSA_REQUIRE(keep_num >= 0 && keep_den >= 1 && keep_num <= keep_den, LSA_ERR_INVALID_ARG,
                "lsa_select_baseline: keep fraction %d/%d outside [0, 1]", keep_num, keep_den);
    const int64_t m_max = ((int64_t)max_old_chunks * keep_num + keep_den / 2) / keep_den;
    LSA_REQUIRE(m_max <= kept_cap, LSA_ERR_CAPACITY,
                "lsa_select_baseline: up to %lld chunks are kept, kept_cap is %d", (long long)m_max, kept_cap);
    const size_t need = lsa_select_baseline_workspace_size(B, max_old_chunks);
    LSA_REQUIRE(ws && ws_bytes >= need, LSA_ERR_WORKSPACE, "lsa_select_baseline: workspace of %zu bytes, %zu needed",
                ws_bytes, need);
    Carver c(ws);
    float *scores = c.take<float>((size_t)B * (max_old_chunks > 0 ? max_old_chunks : 1));
    if (max_old_chunks > 0) {
        random_score_kernel<<<dim3((max_old_chunks + 255) / 256, B), 256, 0, stream>>>(window_start, max_old_chunks,
                                                                                      seed, scores);
        int rc = check_launch("random_score_kernel");
        if (rc) return rc;
    }
    const int nc = cluster_ctas(B), cap = stage_capacity(max_old_chunks, nc);
    if (nc == kTopkCtasOne)
        return launch_topk(random_select_kernel<kTopkCtasOne>, nc, B, cap, stream, "random_select_kernel",
                           (const float *)scores, window_start, max_old_chunks, keep_num, keep_den, kept_idx,
                           kept_count, kept_cap, dev_status, cap);
    return launch_topk(random_select_kernel<kTopkCtas>, nc, B, cap, stream, "random_select_kernel",
                       (const float *)scores, window_start, max_old_chunks, keep_num, keep_den, kept_idx, kept_count,
                       kept_cap, dev_status, cap);
}
