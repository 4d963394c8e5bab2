// pool.cu -- the chunk-slot pools around the decode loop:
//   a5  append of the decoded token to the recent window (the selection made
//       at the window start is reused for 64 steps: gist.science explainer 2.1
//       "Periodische Triggerung", cjcn.com.cn article section 2);
//   a6  fetch of kept cold chunks from the pinned host pool (cjcn.com.cn
//       article section 2; gist.science explainer 2.1 "Dynamisches Fetching").
#include <algorithm>
#include <vector>

#include "block_scan.cuh"
#include "common.cuh"
#include "nvtx_range.cuh"

namespace lsa {

__device__ __forceinline__ void copy_row(uint16_t *dst, const uint16_t *src, int width) {
    // width is a multiple of 8 elements: 16-byte vectors
    for (int c = threadIdx.x; c < width / 8; c += blockDim.x)
        reinterpret_cast<uint4 *>(dst)[c] = reinterpret_cast<const uint4 *>(src)[c];
}

__global__ void append_kernel(const uint16_t *__restrict__ new_k, const uint16_t *__restrict__ new_v,
                              const uint16_t *__restrict__ new_li, uint16_t *__restrict__ k_pool, int64_t k_stride,
                              int k_width, uint16_t *__restrict__ v_pool, int64_t v_stride, int v_width,
                              uint16_t *__restrict__ li_pool, int dl, int64_t n_slots,
                              const int32_t *__restrict__ table, int table_stride,
                              const int32_t *__restrict__ window_start, int32_t *__restrict__ window_len,
                              int32_t *status) {
    __shared__ int64_t s_row;
    const int b = blockIdx.x;
    if (threadIdx.x == 0) {
        const int pos = window_start[b] + window_len[b];
        const int chunk = pos / LSA_CHUNK;
        const int slot = (pos >= 0 && chunk < table_stride) ? table[(size_t)b * table_stride + chunk] : -1;
        s_row = (slot >= 0 && slot < n_slots) ? (int64_t)slot * LSA_CHUNK + pos % LSA_CHUNK : -1;
        if (s_row < 0) flag(status, LSA_DEV_TABLE);
    }
    __syncthreads();
    const int64_t row = s_row;
    if (row < 0) return;
    copy_row(k_pool + row * k_stride, new_k + (size_t)b * k_width, k_width);
    if (v_pool && new_v) copy_row(v_pool + row * v_stride, new_v + (size_t)b * v_width, v_width);
    if (li_pool && new_li) copy_row(li_pool + row * dl, new_li + (size_t)b * dl, dl);
    __syncthreads();
    if (threadIdx.x == 0) window_len[b] += 1;
}

// ---------------------------------------------- device-side residency plan --
// The next window of one sequence needs on the device: its window chunks
// [first_window_chunk, window_end_chunk) (the last one is the chunk its decode
// steps append to) and every kept chunk before the window.  A needed chunk
// that already has a slot in the current table keeps it (the delta against
// what is resident is all that moves); every other needed chunk takes one of
// the slots that the current table leaves free, in ascending chunk and slot
// order.  Chunks that are not needed get -1 in the next table, so their slots
// are free again for the window after.  Needed chunks before the window that
// got a new slot form the copy list, in ascending chunk order.

constexpr int kPlanThreads = 1024;

// One CTA.  ws: used-slot bits [ceil(n_slots / 32)] and the free-slot list [n_need].
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(
    const int32_t *__restrict__ table_cur, int32_t *__restrict__ table_next, int table_len,
    const int32_t *__restrict__ kept_idx, const int32_t *__restrict__ kept_count, int kept_cap, int fw, int fe,
    int n_slots, int32_t *__restrict__ copy_chunk, int32_t *__restrict__ copy_slot, int32_t *__restrict__ copy_count,
    int copy_cap, int32_t *status, uint32_t *__restrict__ used, int32_t *__restrict__ free_list) {
    __shared__ int warp_tot[kPlanThreads / 32 + 1];
    __shared__ int s_need, s_free;
    const int t = threadIdx.x;
    const int words = (n_slots + 31) / 32;
    for (int i = t; i < words; i += kPlanThreads) used[i] = 0u;
    __syncthreads();
    for (int c = t; c < table_len; c += kPlanThreads) {
        const int s = table_cur[c];
        if (s >= 0 && s < n_slots) atomicOr(&used[s >> 5], 1u << (s & 31));
    }
    // needed chunks: table_next first holds 1 for needed, 0 otherwise
    for (int c = t; c < table_len; c += kPlanThreads) table_next[c] = (c >= fw && c < fe) ? 1 : 0;
    __syncthreads();
    const int cnt = min(max(kept_count[0], 0), kept_cap);
    for (int i = t; i < cnt; i += kPlanThreads) {
        const int c = kept_idx[i];
        if (c >= 0 && c < table_len) table_next[c] = 1;
        else flag(status, LSA_DEV_INDEX);
    }
    __syncthreads();
    // rank of every needed chunk without a slot, in chunk order; chunks before fw come first
    int base = 0;
    for (int c0 = 0; c0 < table_len; c0 += kPlanThreads) {
        const int c = c0 + t;
        int needs = 0;
        if (c < table_len) {
            const int s = table_cur[c];
            needs = table_next[c] == 1 && !(s >= 0 && s < n_slots);
        }
        int tot;
        const int r = block_exclusive_scan<kPlanThreads>(needs, warp_tot, &tot);
        if (needs) table_next[c] = -2 - (base + r);   // encodes the rank until slots are known
        base += tot;
    }
    if (t == 0) s_need = base;
    // free slots in ascending order, as many as are needed
    int fbase = 0;
    for (int s0 = 0; s0 < n_slots && fbase < base; s0 += kPlanThreads) {
        const int s = s0 + t;
        const int fr = s < n_slots && !((used[s >> 5] >> (s & 31)) & 1u);
        int tot;
        const int r = block_exclusive_scan<kPlanThreads>(fr, warp_tot, &tot);
        if (fr && fbase + r < base) free_list[fbase + r] = s;
        fbase += tot;
    }
    if (t == 0) s_free = min(fbase, base);
    __syncthreads();
    const int n_free = s_free;
    int cold_new = 0;
    for (int c = t; c < table_len; c += kPlanThreads) {
        const int v = table_next[c];
        int out;
        if (v == 1) out = table_cur[c];                 // needed and resident: keeps its slot
        else if (v <= -2) {
            const int rank = -2 - v;
            out = rank < n_free ? free_list[rank] : -1;
            if (out >= 0 && c < fw) {
                if (rank < copy_cap) {
                    copy_chunk[rank] = c;
                    copy_slot[rank] = out;
                }
                cold_new = max(cold_new, rank + 1);
            }
        } else out = -1;
        table_next[c] = out;
    }
    cold_new = __reduce_max_sync(0xffffffffu, cold_new);
    if ((t & 31) == 0) warp_tot[t >> 5] = cold_new;
    __syncthreads();
    if (t == 0) {
        int m = 0;
        for (int w = 0; w < kPlanThreads / 32; ++w) m = max(m, warp_tot[w]);
        if (s_need > n_free) flag(status, LSA_DEV_CAPACITY);
        if (m > copy_cap) flag(status, LSA_DEV_CAPACITY);
        *copy_count = min(m, copy_cap);
    }
}

// ------------------------------------------------------- chunk fetch kernel --
// Copies listed chunks from the pinned host pools (read through their mapped
// device addresses, over the host link) into device pool slots.  One chunk of
// one pool per loop trip of a CTA; each thread keeps four 16-byte loads in
// flight so that enough reads are outstanding on the link.
constexpr int kMaxPools = 4;
struct FetchPools {
    const uint4 *host[kMaxPools];
    uint4 *dev[kMaxPools];
    int64_t words[kMaxPools];   // 16-byte words per chunk
    int n;
};

__global__ void __launch_bounds__(256) fetch_kernel(const FetchPools pools, const int32_t *__restrict__ copy_chunk,
                                                    const int32_t *__restrict__ copy_slot,
                                                    const int32_t *__restrict__ copy_count, int copy_cap,
                                                    int64_t n_host_chunks, int64_t n_slots, int32_t *status) {
    const int n = min(max(copy_count[0], 0), copy_cap);
    for (int64_t job = blockIdx.x; job < (int64_t)n * pools.n; job += gridDim.x) {
        const int j = (int)(job / pools.n), p = (int)(job % pools.n);
        const int c = copy_chunk[j], s = copy_slot[j];
        if (c < 0 || c >= n_host_chunks || s < 0 || s >= n_slots) {
            if (threadIdx.x == 0 && p == 0) flag(status, LSA_DEV_TABLE);
            continue;
        }
        const int64_t W = pools.words[p];
        const uint4 *src = pools.host[p] + (int64_t)c * W;
        uint4 *dst = pools.dev[p] + (int64_t)s * W;
        int64_t i = threadIdx.x;
        for (; i + 3 * 256 < W; i += 4 * 256) {
            const uint4 a = src[i], b = src[i + 256], d = src[i + 512], e = src[i + 768];
            dst[i] = a; dst[i + 256] = b; dst[i + 512] = d; dst[i + 768] = e;
        }
        for (; i < W; i += 256) dst[i] = src[i];
    }
}

// Moves the window of every sequence forward by `by` tokens and resets its
// length (the start of the next lookahead window).
__global__ void advance_kernel(int32_t *window_start, int32_t *window_len, int B, int by, int len) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) {
        window_start[b] += by;
        window_len[b] = len;
    }
}

}  // namespace lsa

namespace lsa {
bool take_copy_failure();   // host copy failure switch (lsa_test_fail_copy)
}

using namespace lsa;

extern "C" int lsa_append_token(const lsa_bf16 *new_k, const lsa_bf16 *new_v, const lsa_bf16 *new_li,
                                lsa_bf16 *k_pool, int64_t k_row_stride, int k_width, lsa_bf16 *v_pool,
                                int64_t v_row_stride, int v_width, lsa_bf16 *li_pool, int dl, int64_t n_slots,
                                const int32_t *chunk_table, int table_stride, const int32_t *window_start,
                                int32_t *window_len, int B, int32_t *dev_status, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(B > 0 && n_slots > 0 && table_stride > 0, LSA_ERR_INVALID_ARG, "lsa_append_token: bad sizes");
    LSA_REQUIRE(new_k && k_pool && chunk_table && window_start && window_len, LSA_ERR_INVALID_ARG,
                "lsa_append_token: null pointer");
    LSA_REQUIRE(k_width > 0 && k_width % 8 == 0 && k_row_stride >= k_width && k_row_stride % 8 == 0,
                LSA_ERR_INVALID_ARG, "lsa_append_token: k width/stride must be positive multiples of 8");
    LSA_REQUIRE(!v_pool || (new_v && v_width > 0 && v_width % 8 == 0 && v_row_stride >= v_width && v_row_stride % 8 == 0),
                LSA_ERR_INVALID_ARG, "lsa_append_token: v width/stride must be positive multiples of 8");
    LSA_REQUIRE(!li_pool || (new_li && dl > 0 && dl % 8 == 0), LSA_ERR_INVALID_ARG,
                "lsa_append_token: indexer key width must be a positive multiple of 8");
    auto al16 = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
    LSA_REQUIRE(al16(new_k) && al16(k_pool) && al16(new_v) && al16(v_pool) && al16(new_li) && al16(li_pool),
                LSA_ERR_INVALID_ARG, "lsa_append_token: rows are copied in 16-byte vectors: 16-byte aligned bases");
    append_kernel<<<B, 128, 0, stream>>>(new_k, new_v, new_li, k_pool, k_row_stride, k_width, v_pool, v_row_stride,
                                         v_width, li_pool, dl, n_slots, chunk_table, table_stride, window_start,
                                         window_len, dev_status);
    return check_launch("append_kernel");
}

extern "C" int lsa_gather_chunks(int n_pools, const void *const *host_pools, const size_t *chunk_bytes,
                                 void *const *dev_pools, int64_t n_host_chunks, int64_t n_slots,
                                 const int32_t *kept_idx_host, int kept_count_host, int first_window_chunk,
                                 int first_free_slot, int32_t *chunk_table_host, int32_t *chunk_table_dev,
                                 int table_len, lsa_stream_t stream, lsa_event_t done, int *n_fetched) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(n_pools >= 1 && n_pools <= 4 && host_pools && chunk_bytes && dev_pools, LSA_ERR_INVALID_ARG,
                "lsa_gather_chunks: need 1..4 pools with host/device bases and chunk sizes");
    for (int i = 0; i < n_pools; ++i)
        LSA_REQUIRE(host_pools[i] && dev_pools[i] && chunk_bytes[i] > 0, LSA_ERR_INVALID_ARG,
                    "lsa_gather_chunks: pool %d has a null base or zero chunk size", i);
    LSA_REQUIRE(kept_count_host >= 0 && (kept_count_host == 0 || kept_idx_host), LSA_ERR_INVALID_ARG,
                "lsa_gather_chunks: null kept list");
    LSA_REQUIRE(chunk_table_host && chunk_table_dev && table_len > 0 && first_window_chunk >= 0 &&
                    first_window_chunk <= table_len && first_free_slot >= 0,
                LSA_ERR_INVALID_ARG, "lsa_gather_chunks: bad chunk table arguments");
    // validate the whole list before enqueuing anything
    int n_cold = 0, prev = -1;
    for (int j = 0; j < kept_count_host; ++j) {
        const int c = kept_idx_host[j];
        LSA_REQUIRE(c > prev, LSA_ERR_INVALID_ARG, "lsa_gather_chunks: kept list not strictly ascending at %d", j);
        prev = c;
        if (c >= first_window_chunk) continue;
        LSA_REQUIRE(c < n_host_chunks, LSA_ERR_TABLE, "lsa_gather_chunks: chunk %d beyond the host pool (%lld chunks)",
                    c, (long long)n_host_chunks);
        ++n_cold;
    }
    LSA_REQUIRE((int64_t)first_free_slot + n_cold <= n_slots, LSA_ERR_CAPACITY,
                "lsa_gather_chunks: %d chunks do not fit in slots %d..%lld", n_cold, first_free_slot,
                (long long)n_slots - 1);
    // The new entries of the host table are built aside and written only once every chunk
    // copy is enqueued: on an error return the caller's table is as it was.
    std::vector<int32_t> table(chunk_table_host, chunk_table_host + first_window_chunk);
    for (int c = 0; c < first_window_chunk; ++c) table[c] = -1;
    int slot = first_free_slot;
    int j = 0;
    while (j < kept_count_host && kept_idx_host[j] < first_window_chunk) {
        int e = j;
        while (e + 1 < kept_count_host && kept_idx_host[e + 1] < first_window_chunk &&
               kept_idx_host[e + 1] == kept_idx_host[e] + 1)
            ++e;
        const int c0 = kept_idx_host[j], len = e - j + 1;
        for (int i = 0; i < n_pools; ++i) {
            const char *src = static_cast<const char *>(host_pools[i]) + (size_t)c0 * chunk_bytes[i];
            char *dst = static_cast<char *>(dev_pools[i]) + (size_t)slot * chunk_bytes[i];
            if (take_copy_failure()) return fail(LSA_ERR_CUDA, "lsa_gather_chunks: chunk copy failed (injected)");
            LSA_CUDA(cudaMemcpyAsync(dst, src, (size_t)len * chunk_bytes[i], cudaMemcpyHostToDevice, stream));
        }
        for (int r = 0; r < len; ++r) table[c0 + r] = slot + r;
        slot += len;
        j = e + 1;
    }
    std::vector<int32_t> before(chunk_table_host, chunk_table_host + first_window_chunk);
    std::copy(table.begin(), table.end(), chunk_table_host);
    cudaError_t err = take_copy_failure() ? cudaErrorUnknown
                                          : cudaMemcpyAsync(chunk_table_dev, chunk_table_host,
                                                            sizeof(int32_t) * (size_t)table_len,
                                                            cudaMemcpyHostToDevice, stream);
    if (err != cudaSuccess) {
        std::copy(before.begin(), before.end(), chunk_table_host);
        return fail(LSA_ERR_CUDA, "lsa_gather_chunks: chunk table copy failed: %s", cudaGetErrorString(err));
    }
    if (done) LSA_CUDA(cudaEventRecord(done, stream));
    if (n_fetched) *n_fetched = n_cold;
    return LSA_OK;
}

extern "C" size_t lsa_plan_residency_workspace_size(int table_len, int64_t n_slots) {
    if (table_len <= 0 || n_slots <= 0) return 0;
    Carver c(nullptr);
    c.take<uint32_t>((size_t)(n_slots + 31) / 32);
    c.take<int32_t>((size_t)table_len);
    return align_up(c.used, 256);
}

extern "C" int lsa_plan_residency(const int32_t *table_cur, int32_t *table_next, int table_len,
                                  const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
                                  int first_window_chunk, int window_end_chunk, int64_t n_slots, int32_t *copy_chunk,
                                  int32_t *copy_slot, int32_t *copy_count, int copy_cap, int32_t *dev_status, void *ws,
                                  size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(table_cur && table_next && kept_idx && kept_count && copy_chunk && copy_slot && copy_count,
                LSA_ERR_INVALID_ARG, "lsa_plan_residency: null pointer");
    LSA_REQUIRE(table_cur != table_next, LSA_ERR_INVALID_ARG,
                "lsa_plan_residency: the next table must not be the current one");
    LSA_REQUIRE(table_len > 0 && kept_cap > 0 && copy_cap > 0 && n_slots > 0 && n_slots < (int64_t)1 << 30,
                LSA_ERR_INVALID_ARG, "lsa_plan_residency: bad sizes");
    LSA_REQUIRE(first_window_chunk >= 0 && first_window_chunk <= window_end_chunk && window_end_chunk <= table_len,
                LSA_ERR_INVALID_ARG, "lsa_plan_residency: window chunks [%d, %d) outside the table of %d",
                first_window_chunk, window_end_chunk, table_len);
    const size_t need = lsa_plan_residency_workspace_size(table_len, n_slots);
    LSA_REQUIRE(ws && ws_bytes >= need, LSA_ERR_WORKSPACE, "lsa_plan_residency: workspace of %zu bytes, %zu needed",
                ws_bytes, need);
    Carver c(ws);
    uint32_t *used = c.take<uint32_t>((size_t)(n_slots + 31) / 32);
    int32_t *free_list = c.take<int32_t>((size_t)table_len);
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(table_cur, table_next, table_len, kept_idx, kept_count, kept_cap,
                                               first_window_chunk, window_end_chunk, (int)n_slots, copy_chunk,
                                               copy_slot, copy_count, copy_cap, dev_status, used, free_list);
    return check_launch("plan_kernel");
}

extern "C" int lsa_fetch_chunks(int n_pools, const void *const *host_pools, const size_t *chunk_bytes,
                                void *const *dev_pools, int64_t n_host_chunks, int64_t n_slots,
                                const int32_t *copy_chunk, const int32_t *copy_slot, const int32_t *copy_count,
                                int copy_cap, int32_t *dev_status, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(n_pools >= 1 && n_pools <= kMaxPools && host_pools && chunk_bytes && dev_pools, LSA_ERR_INVALID_ARG,
                "lsa_fetch_chunks: need 1..%d pools with host/device bases and chunk sizes", kMaxPools);
    LSA_REQUIRE(copy_chunk && copy_slot && copy_count && copy_cap > 0 && n_host_chunks > 0 && n_slots > 0,
                LSA_ERR_INVALID_ARG, "lsa_fetch_chunks: null copy list or bad sizes");
    FetchPools fp = {};
    fp.n = n_pools;
    for (int i = 0; i < n_pools; ++i) {
        LSA_REQUIRE(host_pools[i] && dev_pools[i] && chunk_bytes[i] > 0 && chunk_bytes[i] % 16 == 0,
                    LSA_ERR_INVALID_ARG, "lsa_fetch_chunks: pool %d needs bases and a chunk size that is a "
                    "positive multiple of 16 bytes", i);
        // The host pool must be page-locked memory that the device can read; its device
        // address comes from the runtime (the same value under unified addressing).
        cudaPointerAttributes at;
        LSA_CUDA(cudaPointerGetAttributes(&at, host_pools[i]));
        LSA_REQUIRE(at.type == cudaMemoryTypeHost && at.devicePointer, LSA_ERR_INVALID_ARG,
                    "lsa_fetch_chunks: host pool %d is not page-locked host memory mapped for the device", i);
        LSA_REQUIRE(((uintptr_t)at.devicePointer & 15) == 0 && ((uintptr_t)dev_pools[i] & 15) == 0,
                    LSA_ERR_INVALID_ARG, "lsa_fetch_chunks: pool %d is not 16-byte aligned", i);
        fp.host[i] = static_cast<const uint4 *>(at.devicePointer);
        fp.dev[i] = static_cast<uint4 *>(dev_pools[i]);
        fp.words[i] = (int64_t)(chunk_bytes[i] / 16);
    }
    fetch_kernel<<<2 * sm_count(), 256, 0, stream>>>(fp, copy_chunk, copy_slot, copy_count, copy_cap, n_host_chunks,
                                                     n_slots, dev_status);
    return check_launch("fetch_kernel");
}

extern "C" int lsa_advance_window(int32_t *window_start, int32_t *window_len, int B, int by, int new_len,
                                  lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(window_start && window_len && B > 0 && by >= 0 && by % LSA_CHUNK == 0 && new_len >= 0,
                LSA_ERR_INVALID_ARG, "lsa_advance_window: bad arguments (B=%d by=%d new_len=%d)", B, by, new_len);
    advance_kernel<<<(B + 255) / 256, 256, 0, stream>>>(window_start, window_len, B, by, new_len);
    return check_launch("advance_kernel");
}
