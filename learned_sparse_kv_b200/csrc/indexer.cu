// indexer.cu -- multi-head indexer scores on tensor cores, shared by
//   a1  the Neural Memory Indexer chunk gate (identity activation, then
//       sigmoid >= 0.5, i.e. logit >= 0) and its order-preserving compaction;
//   a2  the Lightning-Indexer token scores (ReLU activation) over the tokens of
//       kept chunks that lie before the recent window.
// Both compute score(row) = sum_h w_h * act(q_h . key_row) for 64 key rows at a
// time: a [64 x D] . [D x H] product on mma.sync (bf16 in, fp32 accumulate),
// then the activation and the weighted head sum in the epilogue.
// (arXiv 2606.09079 as described by the gist.science explainer 2.1 and the
// cjcn.com.cn article section 2.)
#include "block_scan.cuh"
#include "common.cuh"
#include "nvtx_range.cuh"

namespace lsa {

constexpr int kRows = 64;        // key rows per tile (one chunk of tokens, or 64 chunk keys)
constexpr int kMaxHeads = 128;

struct IdxSmem {
    // keys [64][D] and queries [H][D], rows swizzled in 16-byte chunks
    alignas(128) uint16_t keys[kRows * 128];
    alignas(128) uint16_t q[kMaxHeads * 128];
    float w[kMaxHeads];
    float score[kRows];
};

// Loads q[H][D] (bf16) and w[H] of one sequence into shared memory.
template <int D>
__device__ void load_queries(IdxSmem &sm, const uint16_t *q, const uint16_t *w, int H) {
    constexpr int CPR = D * 2 / 16;  // 16-byte chunks per row
    for (int i = threadIdx.x; i < H * CPR; i += blockDim.x) {
        int r = i / CPR, c = i % CPR;
        cp_async16(reinterpret_cast<char *>(sm.q) + swz(r, c, D * 2), q + (size_t)r * D + c * 8);
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) sm.w[h] = bf16_to_f32(w[h]);
}

// Loads up to 64 key rows; rows >= n_valid are zero-filled.  row_ptr(r) gives the global row.
template <int D, class RowPtr>
__device__ void load_keys(IdxSmem &sm, RowPtr row_ptr, int n_valid) {
    constexpr int CPR = D * 2 / 16;
    for (int i = threadIdx.x; i < kRows * CPR; i += blockDim.x) {
        int r = i / CPR, c = i % CPR;
        const uint16_t *src = r < n_valid ? row_ptr(r) : nullptr;
        void *dst = reinterpret_cast<char *>(sm.keys) + swz(r, c, D * 2);
        if (src)
            cp_async16(dst, src + c * 8);
        else
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
}

// 4 warps: warp i scores rows 16i..16i+15.  Result in sm.score[0..63].
template <int D, bool RELU>
__device__ void score_tile(IdxSmem &sm, int H) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int m0 = warp * 16;
    float acc[kMaxHeads / 8][4];
#pragma unroll
    for (int i = 0; i < kMaxHeads / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    const uint32_t kbase = smem_addr(sm.keys), qbase = smem_addr(sm.q);
#pragma unroll
    for (int kc = 0; kc < D / 8; kc += 2) {
        uint32_t a[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3], kbase + swz(m0 + (lane & 15), kc + (lane >> 4), D * 2));
#pragma unroll
        for (int nt = 0; nt < kMaxHeads / 8; nt += 2) {
            if (nt * 8 < H) {
                uint32_t b0, b1, b2, b3;
                int head = nt * 8 + (lane & 7) + ((lane >> 4) << 3);
                int chunk = kc + ((lane >> 3) & 1);
                ldmatrix_x4(b0, b1, b2, b3, qbase + swz(head, chunk, D * 2));
                mma_bf16_16816(acc[nt], a, b0, b1);
                if ((nt + 1) * 8 < H) mma_bf16_16816(acc[nt + 1], a, b2, b3);
            }
        }
    }
    const int g = lane >> 2, qd = lane & 3;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < kMaxHeads / 8; ++nt) {
        if (nt * 8 < H) {
            float w0 = sm.w[nt * 8 + 2 * qd], w1 = sm.w[nt * 8 + 2 * qd + 1];
            float v0 = acc[nt][0], v1 = acc[nt][1], v2 = acc[nt][2], v3 = acc[nt][3];
            if (RELU) {
                v0 = fmaxf(v0, 0.f); v1 = fmaxf(v1, 0.f); v2 = fmaxf(v2, 0.f); v3 = fmaxf(v3, 0.f);
            }
            s0 += w0 * v0 + w1 * v1;
            s1 += w0 * v2 + w1 * v3;
        }
    }
    s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
    s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
    if (qd == 0) {
        sm.score[m0 + g] = s0;
        sm.score[m0 + g + 8] = s1;
    }
}

// ------------------------------------------------------------------- a1 ----

// Up to four independent indexers gated together (OR mode): indexer i has its
// own queries, head weights and compressed keys, and optional logits output.
constexpr int kMaxIndexers = 4;
struct NmiSet {
    const uint16_t *q[kMaxIndexers];
    const uint16_t *w[kMaxIndexers];
    const uint16_t *khat[kMaxIndexers];
    float *logits[kMaxIndexers];
};

// grid (tiles of 64 chunks, B, indexers).  Writes logits and one 64-bit gate
// mask per tile; indexer i's masks start at masks + i * B * tiles_per_seq.
template <int D>
__global__ void __launch_bounds__(128) nmi_score_kernel(const NmiSet set, const int64_t *__restrict__ off, int H,
                                                        int tiles_per_seq, unsigned long long *__restrict__ masks) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    IdxSmem &sm = *reinterpret_cast<IdxSmem *>(smem_raw);
    const int b = blockIdx.y, tile = blockIdx.x, ix = blockIdx.z;
    const uint16_t *__restrict__ q = set.q[ix];
    const uint16_t *__restrict__ w = set.w[ix];
    const uint16_t *__restrict__ khat = set.khat[ix];
    float *__restrict__ logits = set.logits[ix];
    masks += (size_t)ix * gridDim.y * tiles_per_seq;
    const int64_t first = off[b];
    const int64_t n_ch = off[b + 1] - first;
    const int64_t s0 = (int64_t)tile * kRows;
    if (s0 >= n_ch) {
        if (threadIdx.x == 0) masks[(size_t)b * tiles_per_seq + tile] = 0ull;
        return;
    }
    const int n_valid = (int)(n_ch - s0 < kRows ? n_ch - s0 : kRows);
    load_queries<D>(sm, q + (size_t)b * H * D, w + (size_t)b * H, H);
    load_keys<D>(sm, [&](int r) { return khat + (size_t)(first + s0 + r) * D; }, n_valid);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    score_tile<D, false>(sm, H);
    __syncthreads();
    __shared__ unsigned halves[2];
    const int r = threadIdx.x;
    bool keep = false;
    if (r < kRows) {
        float l = sm.score[r];
        keep = r < n_valid && l >= 0.f;  // sigmoid(l) >= 0.5  <=>  l >= 0
        if (r < n_valid && logits) logits[first + s0 + r] = l;
    }
    unsigned bits = __ballot_sync(0xffffffffu, keep);  // warp 0: rows 0..31, warp 1: rows 32..63
    if ((r & 31) == 0 && r < kRows) halves[r >> 5] = bits;
    __syncthreads();
    if (r == 0)
        masks[(size_t)b * tiles_per_seq + tile] = (unsigned long long)halves[0] | ((unsigned long long)halves[1] << 32);
}

// grid B, 256 threads: gate masks -> ascending kept list, count, capacity flag.
// With several indexers a chunk is kept when any of their masks has its bit.
__global__ void __launch_bounds__(256) nmi_compact_kernel(const unsigned long long *__restrict__ masks, int n_idx,
                                                          const int64_t *__restrict__ off, int tiles_per_seq,
                                                          int32_t *__restrict__ kept_idx, int32_t *__restrict__ kept_count,
                                                          int kept_cap, int32_t *status) {
    __shared__ int warp_tot[256 / 32 + 1];
    const int b = blockIdx.x;
    const int64_t n_ch = off[b + 1] - off[b];
    int n_words = (int)((n_ch + kRows - 1) / kRows);
    if (n_words > tiles_per_seq) {  // more chunks than the host-declared maximum: score only those
        n_words = tiles_per_seq;
        if (threadIdx.x == 0) flag(status, LSA_DEV_INDEX);
    }
    const int per = (n_words + 255) / 256;
    const int w0 = min(n_words, (int)threadIdx.x * per), w1 = min(n_words, w0 + per);
    const unsigned long long *m = masks + (size_t)b * tiles_per_seq;
    const size_t idx_stride = (size_t)gridDim.x * tiles_per_seq;
    auto word = [&](int i) {
        unsigned long long x = m[i];
        for (int j = 1; j < n_idx; ++j) x |= m[j * idx_stride + i];
        return x;
    };
    int mine = 0;
    for (int i = w0; i < w1; ++i) mine += __popcll(word(i));
    int total;
    int pos = block_exclusive_scan<256>(mine, warp_tot, &total);
    int32_t *out = kept_idx + (size_t)b * kept_cap;
    for (int i = w0; i < w1; ++i) {
        unsigned long long bits = word(i);
        while (bits) {
            int bit = __ffsll((long long)bits) - 1;
            bits &= bits - 1;
            if (pos < kept_cap) out[pos] = i * kRows + bit;
            ++pos;
        }
    }
    for (int j = total + threadIdx.x; j < kept_cap; j += 256) out[j] = -1;
    if (threadIdx.x == 0) {
        kept_count[b] = min(total, kept_cap);
        if (total > kept_cap) flag(status, LSA_DEV_CAPACITY);
    }
}

// ------------------------------------------------------------------- a2 ----

// grid (G, B): CTA x of sequence b scores kept cold chunks x, x+G, ...
template <int D>
__global__ void __launch_bounds__(128) li_score_kernel(const uint16_t *__restrict__ q_li, const uint16_t *__restrict__ w_li,
                                                       const uint16_t *__restrict__ li_pool, int64_t n_slots,
                                                       const int32_t *__restrict__ table, int table_stride,
                                                       const int32_t *__restrict__ kept_idx,
                                                       const int32_t *__restrict__ cold, int kept_cap, int H,
                                                       float *__restrict__ scores, int32_t *status) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    IdxSmem &sm = *reinterpret_cast<IdxSmem *>(smem_raw);
    const int b = blockIdx.y;
    const int32_t *kept = kept_idx + (size_t)b * kept_cap;
    const int n_cold = cold[b];
    if ((int)blockIdx.x >= n_cold) return;
    load_queries<D>(sm, q_li + (size_t)b * H * D, w_li + (size_t)b * H, H);
    const int32_t *trow = table + (size_t)b * table_stride;
    float *out = scores + (size_t)b * kept_cap * kRows;
    for (int j = blockIdx.x; j < n_cold; j += gridDim.x) {
        const int chunk = kept[j];
        int slot = (chunk >= 0 && chunk < table_stride) ? trow[chunk] : -1;
        const bool ok = slot >= 0 && slot < n_slots;
        if (!ok && threadIdx.x == 0) flag(status, LSA_DEV_TABLE);
        load_keys<D>(sm, [&](int r) { return li_pool + ((size_t)slot * kRows + r) * D; }, ok ? kRows : 0);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        score_tile<D, true>(sm, H);
        __syncthreads();
        if (threadIdx.x < kRows) out[(size_t)j * kRows + threadIdx.x] = ok ? sm.score[threadIdx.x] : -INFINITY;
        __syncthreads();
    }
}

// ------------------------------------------------------------ host launch --

static bool heads_ok(int H) { return H >= 8 && H <= kMaxHeads && H % 8 == 0; }

namespace li2 {
bool shape_ok(int H, int D, int B);
int launch(const uint16_t *q_li, const uint16_t *w_li, const uint16_t *li_pool, int64_t n_slots, const int32_t *table,
           int table_stride, const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
           const int32_t *window_start, int32_t *cold, int B, int H, int D, float *scores, int32_t *status,
           cudaStream_t stream, const AppendArgs *app);
}  // namespace li2

// True when the indexer kernel for this shape counts the kept cold chunks itself
// (the tcgen05 kernel does, in its prologue); otherwise they are counted first.
bool indexer_counts_cold(int H, int D, int B) { return li2::shape_ok(H, D, B); }

// app (optional, tcgen05 shapes only): the decoded token's rows, appended by the same launch.
int launch_li_scores(const uint16_t *q_li, const uint16_t *w_li, const uint16_t *li_pool, int64_t n_slots,
                     const int32_t *table, int table_stride, const int32_t *kept_idx, const int32_t *kept_count,
                     int kept_cap, const int32_t *window_start, int32_t *cold, int B, int H, int D,
                     float *scores, int32_t *status, cudaStream_t stream, const AppendArgs *app) {
    // Head counts of 32, 64 or 128 run on tcgen05 (M = 128 tokens, N = heads); others on mma.sync.
    if (li2::shape_ok(H, D, B))
        return li2::launch(q_li, w_li, li_pool, n_slots, table, table_stride, kept_idx, kept_count, kept_cap,
                           window_start, cold, B, H, D, scores, status, stream, app);
    if (app) return fail(LSA_ERR_SHAPE, "append with the indexer: only the tcgen05 indexer shapes");
    const size_t smem = sizeof(IdxSmem);
    int per_seq = (sm_count() * 8 + B - 1) / B;
    per_seq = max(1, min(per_seq, kept_cap));
    dim3 grid(per_seq, B);
    if (D == 128) {
        cudaFuncSetAttribute(li_score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        li_score_kernel<128><<<grid, 128, smem, stream>>>(q_li, w_li, li_pool, n_slots, table, table_stride, kept_idx,
                                                          cold, kept_cap, H, scores, status);
    } else {
        cudaFuncSetAttribute(li_score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        li_score_kernel<64><<<grid, 128, smem, stream>>>(q_li, w_li, li_pool, n_slots, table, table_stride, kept_idx,
                                                         cold, kept_cap, H, scores, status);
    }
    return check_launch("li_score_kernel");
}

bool indexer_shape_ok(int H, int D) { return heads_ok(H) && (D == 64 || D == 128); }

}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_nmi_select_union_workspace_size(int n_idx, int B, int max_chunks_per_seq) {
    if (n_idx < 1 || n_idx > kMaxIndexers || B <= 0 || max_chunks_per_seq < 0) return 0;
    Carver c(nullptr);
    int tiles = (max_chunks_per_seq + kRows - 1) / kRows;
    c.take<unsigned long long>((size_t)n_idx * B * (tiles > 0 ? tiles : 1));
    return align_up(c.used, 256);
}

extern "C" size_t lsa_nmi_select_workspace_size(int B, int max_chunks_per_seq) {
    return lsa_nmi_select_union_workspace_size(1, B, max_chunks_per_seq);
}

namespace lsa {

static int nmi_select_impl(const char *who, int n_idx, const NmiSet &set, const int64_t *seq_chunk_offset, int B,
                           int Hn, int dn, int64_t total_chunks, int max_chunks_per_seq, int32_t *kept_idx,
                           int32_t *kept_count, int kept_cap, int32_t *dev_status, void *ws, size_t ws_bytes,
                           cudaStream_t stream) {
    LSA_REQUIRE(B > 0, LSA_ERR_INVALID_ARG, "%s: B must be positive (got %d)", who, B);
    for (int i = 0; i < n_idx; ++i)
        LSA_REQUIRE(set.q[i] && set.w[i] && set.khat[i], LSA_ERR_INVALID_ARG, "%s: null input pointer of indexer %d",
                    who, i);
    LSA_REQUIRE(seq_chunk_offset && kept_idx && kept_count, LSA_ERR_INVALID_ARG, "%s: null input or output pointer",
                who);
    LSA_REQUIRE(indexer_shape_ok(Hn, dn), LSA_ERR_SHAPE,
                "%s: unsupported Hn=%d dn=%d (dn in {64,128}, Hn multiple of 8 up to 128)", who, Hn, dn);
    LSA_REQUIRE(max_chunks_per_seq >= 0 && total_chunks >= 0 && kept_cap >= 1, LSA_ERR_INVALID_ARG,
                "%s: bad sizes (max_chunks_per_seq=%d total_chunks=%lld kept_cap=%d)", who, max_chunks_per_seq,
                (long long)total_chunks, kept_cap);
    const size_t need = lsa_nmi_select_union_workspace_size(n_idx, B, max_chunks_per_seq);
    LSA_REQUIRE(ws_bytes >= need && ws, LSA_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", who, ws_bytes,
                need);
    const int tiles = max(1, (max_chunks_per_seq + kRows - 1) / kRows);
    Carver c(ws);
    auto *masks = c.take<unsigned long long>((size_t)n_idx * B * tiles);
    const size_t smem = sizeof(IdxSmem);
    dim3 grid(tiles, B, n_idx);
    if (dn == 128) {
        LSA_CUDA(cudaFuncSetAttribute(nmi_score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        nmi_score_kernel<128><<<grid, 128, smem, stream>>>(set, seq_chunk_offset, Hn, tiles, masks);
    } else {
        LSA_CUDA(cudaFuncSetAttribute(nmi_score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        nmi_score_kernel<64><<<grid, 128, smem, stream>>>(set, seq_chunk_offset, Hn, tiles, masks);
    }
    int rc = check_launch("nmi_score_kernel");
    if (rc) return rc;
    nmi_compact_kernel<<<B, 256, 0, stream>>>(masks, n_idx, seq_chunk_offset, tiles, kept_idx, kept_count, kept_cap,
                                              dev_status);
    return check_launch("nmi_compact_kernel");
}

}  // namespace lsa

extern "C" int lsa_nmi_select(const lsa_bf16 *q, const lsa_bf16 *w, const lsa_bf16 *khat,
                              const int64_t *seq_chunk_offset, int B, int Hn, int dn, int64_t total_chunks,
                              int max_chunks_per_seq, int32_t *kept_idx, int32_t *kept_count, int kept_cap,
                              float *logits, int32_t *dev_status, void *ws, size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    NmiSet set = {};
    set.q[0] = q; set.w[0] = w; set.khat[0] = khat; set.logits[0] = logits;
    return nmi_select_impl("lsa_nmi_select", 1, set, seq_chunk_offset, B, Hn, dn, total_chunks, max_chunks_per_seq,
                           kept_idx, kept_count, kept_cap, dev_status, ws, ws_bytes, stream);
}

extern "C" int lsa_nmi_select_union(int n_idx, const lsa_bf16 *const *q, const lsa_bf16 *const *w,
                                    const lsa_bf16 *const *khat, const int64_t *seq_chunk_offset, int B, int Hn, int dn,
                                    int64_t total_chunks, int max_chunks_per_seq, int32_t *kept_idx,
                                    int32_t *kept_count, int kept_cap, float *logits, int32_t *dev_status, void *ws,
                                    size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(n_idx >= 1 && n_idx <= kMaxIndexers, LSA_ERR_INVALID_ARG,
                "lsa_nmi_select_union: n_idx must be 1..%d (got %d)", kMaxIndexers, n_idx);
    LSA_REQUIRE(q && w && khat, LSA_ERR_INVALID_ARG, "lsa_nmi_select_union: null pointer array");
    NmiSet set = {};
    for (int i = 0; i < n_idx; ++i) {
        set.q[i] = q[i]; set.w[i] = w[i]; set.khat[i] = khat[i];
        set.logits[i] = logits ? logits + (size_t)i * total_chunks : nullptr;
    }
    return nmi_select_impl("lsa_nmi_select_union", n_idx, set, seq_chunk_offset, B, Hn, dn, total_chunks,
                           max_chunks_per_seq, kept_idx, kept_count, kept_cap, dev_status, ws, ws_bytes, stream);
}
