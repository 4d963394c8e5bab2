// pool.cu -- the chunk-slot pools around the decode loop:
//   a5  append of the decoded token to the recent window (the selection made
//       at the window start is reused for 64 steps: gist.science explainer 2.1
//       "Periodische Triggerung", cjcn.com.cn article section 2);
//   a6  fetch of kept cold chunks from the pinned host pool (cjcn.com.cn
//       article section 2; gist.science explainer 2.1 "Dynamisches Fetching").
#include <vector>

#include "common.cuh"

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

}  // namespace lsa

using namespace lsa;

extern "C" int lsa_append_token(const lsa_bf16 *new_k, const lsa_bf16 *new_v, const lsa_bf16 *new_li,
                                lsa_bf16 *k_pool, int64_t k_row_stride, int k_width, lsa_bf16 *v_pool,
                                int64_t v_row_stride, int v_width, lsa_bf16 *li_pool, int dl, int64_t n_slots,
                                const int32_t *chunk_table, int table_stride, const int32_t *window_start,
                                int32_t *window_len, int B, int32_t *dev_status, lsa_stream_t stream) {
    LSA_REQUIRE(B > 0 && n_slots > 0 && table_stride > 0, LSA_ERR_INVALID_ARG, "lsa_append_token: bad sizes");
    LSA_REQUIRE(new_k && k_pool && chunk_table && window_start && window_len, LSA_ERR_INVALID_ARG,
                "lsa_append_token: null pointer");
    LSA_REQUIRE(k_width > 0 && k_width % 8 == 0 && k_row_stride >= k_width && k_row_stride % 8 == 0,
                LSA_ERR_INVALID_ARG, "lsa_append_token: k width/stride must be positive multiples of 8");
    LSA_REQUIRE(!v_pool || (new_v && v_width > 0 && v_width % 8 == 0 && v_row_stride >= v_width && v_row_stride % 8 == 0),
                LSA_ERR_INVALID_ARG, "lsa_append_token: v width/stride must be positive multiples of 8");
    LSA_REQUIRE(!li_pool || (new_li && dl > 0 && dl % 8 == 0), LSA_ERR_INVALID_ARG,
                "lsa_append_token: indexer key width must be a positive multiple of 8");
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
    for (int c = 0; c < first_window_chunk; ++c) chunk_table_host[c] = -1;
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
            LSA_CUDA(cudaMemcpyAsync(dst, src, (size_t)len * chunk_bytes[i], cudaMemcpyHostToDevice, stream));
        }
        for (int r = 0; r < len; ++r) chunk_table_host[c0 + r] = slot + r;
        slot += len;
        j = e + 1;
    }
    LSA_CUDA(cudaMemcpyAsync(chunk_table_dev, chunk_table_host, sizeof(int32_t) * (size_t)table_len,
                             cudaMemcpyHostToDevice, stream));
    if (done) LSA_CUDA(cudaEventRecord(done, stream));
    if (n_fetched) *n_fetched = n_cold;
    return LSA_OK;
}
