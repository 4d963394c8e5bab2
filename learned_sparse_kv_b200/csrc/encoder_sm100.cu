// encoder_sm100.cu -- the memory indexer's query encoder on 5th-generation tensor
// cores: the hidden state h_t of each token is projected down to the low rank
// (2048 in the pages' configuration), then up to the indexer's query heads,
// and the per-head weights are projected from h_t directly.
// (arXiv 2606.09079: the indexer maps h_t to low-rank indexer queries, gist.science
// explainer 2.1; only these low-rank projections are trained, 2.3; rank 2048,
// cjcn.com.cn article section 4.)
//
//   c = W_down h      q = W_up c      w = W_head h        (weights [out, in], bf16)
//
// Each product is Y[B, N] = X[B, K] . W[N, K]^T with a few tokens B and many
// weight rows N, so it streams the weights once from HBM.  It runs "swapped":
// the tensor-core M dimension is 128 weight rows, N is the tokens padded to a
// multiple of 32 (TMA fills the rows past B with zeros), K is streamed in blocks
// of 64 columns through a 4-stage TMA ring (96 KB of shared memory, so two CTAs
// share a multiprocessor).  The grid is (row tiles, K splits) with about two
// CTAs per multiprocessor streaming weights at once; every CTA
// writes an fp32 partial [split][token][row] and a reduce kernel sums the
// splits in a fixed order (no atomics: the result does not depend on timing).
// The second product takes c as two bf16 operands, hi = bf16(c) and
// lo = bf16(c - hi), stacked as token rows 0..T-1 and T..2T-1 of one operand:
// one MMA computes W_up.hi and W_up.lo side by side, and the epilogue adds the
// two, so c enters with about 16 significant bits instead of 8.
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 0..3 epilogue.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "nvtx_range.cuh"
#include "sm100.cuh"

namespace lsa {
namespace enc {

using namespace sm100;

constexpr int THREADS = 128;
constexpr int STAGES = 4;
constexpr int MAX_N = 64;                  // token columns of one MMA (padded tokens, both parts)
constexpr int MAX_B = MAX_N / 2;           // tokens per call
constexpr uint32_t A_BYTES = 128 * 128;    // 128 weight rows x 64 columns
constexpr uint32_t X_BYTES = MAX_N * 128;  // up to 64 token rows x 64 columns (96 KB per CTA: two per SM)

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_BYTES];
    uint8_t x[STAGES][X_BYTES];
    uint64_t full[STAGES], empty[STAGES];
    uint64_t acc_full;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    float *partial;     // [splits][B][n_rows]
    int32_t *status;
    int n_rows;         // weight rows (output entries per token)
    int kb_total;       // 64-column blocks of K
    int kb_per_split;
    int B;              // tokens
    int n_cols;         // MMA N: padded tokens (x2 when two_part)
    int two_part;       // X rows T..2T-1 hold the lo part of rows 0..T-1 (T = n_cols / 2)
    uint32_t x_bytes;   // bytes of one X stage that TMA writes (n_cols x 128)
};

__device__ __forceinline__ void umma1(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(uint32_t(acc)));
}
__device__ __forceinline__ void commit1(const uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tma2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
            smem_addr(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void expect_tx1(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool wait_or_abort(Smem &sm, const uint64_t *bar, uint32_t parity, int32_t *status) {
    if (sm.abort_flag) return false;
    if (mbar_wait(bar, parity, WAIT_NS)) return true;
    sm.abort_flag = 1;
    flag(status, LSA_DEV_TIMEOUT);
    return false;
}

// grid (ceil(n_rows / 128), splits)
__global__ void __launch_bounds__(THREADS) skinny_gemm_kernel(const __grid_constant__ CUtensorMap w_map,
                                                              const __grid_constant__ CUtensorMap x_map,
                                                              const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * 128, split = blockIdx.y;
    const int kb0 = split * p.kb_per_split, kb1 = min(p.kb_total, kb0 + p.kb_per_split);
    const int n_kb = max(0, kb1 - kb0);
    const uint32_t tmem_cols = p.n_cols <= 32 ? 32u : 64u;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&sm.full[i], 1); mbar_init(&sm.empty[i], 1); }
        mbar_init(&sm.acc_full, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&sm.tmem_base)),
                     "r"(tmem_cols));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    int issued = 0;   // loads issued by the producer (lane 0 of warp 0)
    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        for (int i = 0; i < n_kb; ++i) {
            const int s = i % STAGES;
            if (i >= STAGES && !wait_or_abort(sm, &sm.empty[s], ((i / STAGES) - 1) & 1, p.status)) break;
            expect_tx1(&sm.full[s], A_BYTES + p.x_bytes);
            tma2d(sm.a[s], &w_map, 64 * (kb0 + i), m0, &sm.full[s]);
            tma2d(sm.x[s], &x_map, 64 * (kb0 + i), 0, &sm.full[s]);
            ++issued;
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16_f32(128, p.n_cols, false, false);
        for (int i = 0; i < n_kb; ++i) {
            const int s = i % STAGES;
            if (!wait_or_abort(sm, &sm.full[s], (i / STAGES) & 1, p.status)) break;
            tc_fence_after();
            const uint64_t ad = smem_desc_sw128(smem_addr(sm.a[s]), 16, 1024);
            const uint64_t xd = smem_desc_sw128(smem_addr(sm.x[s]), 16, 1024);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) umma1(tmem, ad + 2 * k4, xd + 2 * k4, idesc, (i | k4) != 0);
            commit1(&sm.empty[s]);
        }
        commit1(&sm.acc_full);   // arrives once every MMA issued above has completed
    }
    __syncwarp();

    // ---------------------------------------------------- epilogue (4 warps)
    const bool ok = mbar_wait(&sm.acc_full, 0, WAIT_NS);
    if (!ok && lane == 0) {
        sm.abort_flag = 1;
        flag(p.status, LSA_DEV_TIMEOUT);
    }
    tc_fence_after();
    const int row = m0 + 32 * warp + lane;                  // TMEM lane = weight row
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const int T = p.two_part ? p.n_cols / 2 : p.n_cols;
    const bool any = n_kb > 0 && ok && sm.abort_flag == 0;
    for (int c0 = 0; c0 < T; c0 += 32) {
        uint32_t v[32], v2[32];
        tmem_ld32(tmem + lane_base + c0, v);
        if (p.two_part) tmem_ld32(tmem + lane_base + T + c0, v2);
        tmem_wait_ld();
        if (row < p.n_rows) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int b = c0 + i;
                if (b < p.B) {
                    float y = any ? __uint_as_float(v[i]) : 0.f;
                    if (p.two_part && any) y += __uint_as_float(v2[i]);
                    p.partial[((size_t)split * p.B + b) * p.n_rows + row] = y;
                }
            }
        }
    }
    // Loads still in flight after an abort land before the CTA leaves: the
    // producer waits for the last `issued` loads' full barriers (each bounded).
    if (warp == 0 && lane == 0 && sm.abort_flag) {
        for (int i = max(0, issued - STAGES); i < issued; ++i)
            (void)mbar_wait(&sm.full[i % STAGES], (i / STAGES) & 1, WAIT_NS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
}

// Sums the splits of c = W_down h and writes it as the two stacked bf16 parts
// of the next product's operand: rows 0..T-1 hi, rows T..2T-1 lo (zero past B).
__global__ void __launch_bounds__(256) reduce_split_kernel(const float *__restrict__ partial, int splits, int B,
                                                           int n_rows, int T, uint16_t *__restrict__ x2) {
    const int r = blockIdx.x * 256 + threadIdx.x, b = blockIdx.y;   // b < T
    if (r >= n_rows) return;
    float c = 0.f;
    if (b < B)
        for (int s = 0; s < splits; ++s) c += partial[((size_t)s * B + b) * n_rows + r];
    const __nv_bfloat16 hi = __float2bfloat16_rn(c);
    const __nv_bfloat16 lo = __float2bfloat16_rn(c - __bfloat162float(hi));
    x2[(size_t)b * n_rows + r] = *reinterpret_cast<const uint16_t *>(&hi);
    x2[(size_t)(T + b) * n_rows + r] = *reinterpret_cast<const uint16_t *>(&lo);
}

// Sums the splits of a final output and writes it as bf16 (and fp32 if asked).
__global__ void __launch_bounds__(256) reduce_out_kernel(const float *__restrict__ partial, int splits, int B,
                                                         int n_rows, uint16_t *__restrict__ out_bf16,
                                                         float *__restrict__ out_f32) {
    const int r = blockIdx.x * 256 + threadIdx.x, b = blockIdx.y;
    if (r >= n_rows) return;
    float y = 0.f;
    for (int s = 0; s < splits; ++s) y += partial[((size_t)s * B + b) * n_rows + r];
    const __nv_bfloat16 v = __float2bfloat16_rn(y);
    out_bf16[(size_t)b * n_rows + r] = *reinterpret_cast<const uint16_t *>(&v);
    if (out_f32) out_f32[(size_t)b * n_rows + r] = y;
}

// --------------------------------------------------------------- host side --

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [rows, cols] bf16 row-major, box {64 columns, box_rows}, 128-byte swizzle, zero fill outside.
static bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiled>(ptr);
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int pad32(int b) { return (b + 31) / 32 * 32; }

// K splits so that the grid is about two CTAs per multiprocessor.
static int kb_per_split(int row_tiles, int kb_total) {
    const int want = max(1, (2 * sm_count() + row_tiles - 1) / row_tiles);
    const int splits = min(kb_total, want);
    return (kb_total + splits - 1) / splits;
}

struct Plan {
    int row_tiles, kbs, splits;
};
static Plan plan(int n_rows, int K) {
    Plan pl;
    pl.row_tiles = (n_rows + 127) / 128;
    const int kb_total = K / 64;
    pl.kbs = kb_per_split(pl.row_tiles, kb_total);
    pl.splits = (kb_total + pl.kbs - 1) / pl.kbs;
    return pl;
}

size_t smem_bytes() { return sizeof(Smem) + 1024; }

static int gemm(const uint16_t *w, int n_rows, int K, const uint16_t *x, int x_rows, int B, int n_cols,
                bool two_part, float *partial, const Plan &pl, int32_t *status, cudaStream_t stream) {
    CUtensorMap w_map, x_map;
    if (!make_map(&w_map, w, (uint64_t)K, (uint64_t)n_rows, 128) ||
        !make_map(&x_map, x, (uint64_t)K, (uint64_t)x_rows, (uint32_t)n_cols))
        return fail(LSA_ERR_CUDA, "lsa_query_encoder: cuTensorMapEncodeTiled failed");
    Params prm;
    prm.partial = partial; prm.status = status; prm.n_rows = n_rows; prm.kb_total = K / 64;
    prm.kb_per_split = pl.kbs; prm.B = B; prm.n_cols = n_cols; prm.two_part = two_part ? 1 : 0;
    prm.x_bytes = (uint32_t)n_cols * 128;
    const size_t smem = smem_bytes();
    LSA_CUDA(cudaFuncSetAttribute(skinny_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    skinny_gemm_kernel<<<dim3(pl.row_tiles, pl.splits), THREADS, smem, stream>>>(w_map, x_map, prm);
    return check_launch("skinny_gemm_kernel");
}

}  // namespace enc
}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_query_encoder_workspace_size(int B, int d_model, int rank, int Hn, int dn) {
    if (B <= 0 || B > enc::MAX_B || d_model <= 0 || rank <= 0 || Hn <= 0 || dn <= 0) return 0;
    const enc::Plan p1 = enc::plan(rank, d_model), p2 = enc::plan(Hn * dn, rank), p3 = enc::plan(Hn, d_model);
    const size_t part = std::max({(size_t)p1.splits * B * rank, (size_t)p2.splits * B * Hn * dn,
                                  (size_t)p3.splits * B * Hn});
    Carver c(nullptr);
    c.take<float>(part);                                         // split partials (reused by each product)
    c.take<uint16_t>((size_t)2 * enc::pad32(B) * rank);          // c as stacked hi / lo bf16 rows
    return align_up(c.used, 256);
}

extern "C" int lsa_query_encoder(const lsa_bf16 *h, int B, int d_model, const lsa_bf16 *w_down, int rank,
                                 const lsa_bf16 *w_up, const lsa_bf16 *w_head, int Hn, int dn, lsa_bf16 *q_out,
                                 lsa_bf16 *w_out, float *q_f32, float *w_f32, int32_t *dev_status, void *ws,
                                 size_t ws_bytes, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(h && w_down && w_up && w_head && q_out && w_out, LSA_ERR_INVALID_ARG,
                "lsa_query_encoder: null pointer");
    LSA_REQUIRE(B >= 1 && B <= enc::MAX_B, LSA_ERR_SHAPE, "lsa_query_encoder: B=%d outside [1, %d]", B, enc::MAX_B);
    LSA_REQUIRE(d_model >= 64 && d_model % 64 == 0 && rank >= 64 && rank % 64 == 0, LSA_ERR_SHAPE,
                "lsa_query_encoder: d_model=%d and rank=%d must be positive multiples of 64", d_model, rank);
    LSA_REQUIRE(Hn >= 1 && dn >= 1 && (int64_t)Hn * dn <= (1 << 20), LSA_ERR_SHAPE,
                "lsa_query_encoder: bad head shape Hn=%d dn=%d", Hn, dn);
    const size_t need = lsa_query_encoder_workspace_size(B, d_model, rank, Hn, dn);
    LSA_REQUIRE(ws && ws_bytes >= need, LSA_ERR_WORKSPACE, "lsa_query_encoder: workspace of %zu bytes, %zu needed",
                ws_bytes, need);
    const enc::Plan p1 = enc::plan(rank, d_model), p2 = enc::plan(Hn * dn, rank), p3 = enc::plan(Hn, d_model);
    const size_t part_n = std::max({(size_t)p1.splits * B * rank, (size_t)p2.splits * B * Hn * dn,
                                    (size_t)p3.splits * B * Hn});
    Carver c(ws);
    float *partial = c.take<float>(part_n);
    const int T = enc::pad32(B);
    uint16_t *x2 = c.take<uint16_t>((size_t)2 * T * rank);
    // w = W_head h
    int rc = enc::gemm(w_head, Hn, d_model, h, B, B, T, false, partial, p3, dev_status, stream);
    if (rc) return rc;
    enc::reduce_out_kernel<<<dim3((Hn + 255) / 256, B), 256, 0, stream>>>(partial, p3.splits, B, Hn, w_out, w_f32);
    if ((rc = check_launch("reduce_out_kernel"))) return rc;
    // c = W_down h, kept as bf16 hi + lo
    if ((rc = enc::gemm(w_down, rank, d_model, h, B, B, T, false, partial, p1, dev_status, stream))) return rc;
    enc::reduce_split_kernel<<<dim3((rank + 255) / 256, T), 256, 0, stream>>>(partial, p1.splits, B, rank, T, x2);
    if ((rc = check_launch("reduce_split_kernel"))) return rc;
    // q = W_up c = W_up hi + W_up lo
    if ((rc = enc::gemm(w_up, Hn * dn, rank, x2, 2 * T, B, 2 * T, true, partial, p2, dev_status, stream))) return rc;
    enc::reduce_out_kernel<<<dim3((Hn * dn + 255) / 256, B), 256, 0, stream>>>(partial, p2.splits, B, Hn * dn, q_out,
                                                                                q_f32);
    return check_launch("reduce_out_kernel");
}
