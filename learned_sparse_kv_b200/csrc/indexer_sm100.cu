// indexer_sm100.cu -- a2 on 5th-generation tensor cores: Lightning-Indexer token
// scores over the tokens of kept chunks that lie before the recent window.
// (arXiv 2606.09079: the native indexer's finer top-k inside the fetched set,
// gist.science explainer 2.1 "Gestufte Selektion"; cjcn.com.cn article section 2.)
//
//   score(t) = sum_h w_h * max(0, q_h . key_t)
//
// Persistent CTAs walk contiguous ranges of "tiles": two consecutive kept cold
// chunks of one sequence = 128 tokens.  Per tile one tcgen05.mma chain computes
// D[128 tokens x H heads] = keys[128 x dl] . q^T[dl x H] into tensor memory
// (M = 128, N = H, K = dl in steps of 16); an epilogue warpgroup reads one
// token row per thread, applies ReLU and the head weights, and writes the
// score.  Keys arrive by TMA tile loads of whole chunk slots (64 rows x 64
// columns, 128-byte swizzle) into a 3-stage ring; the per-sequence query heads
// live in two buffers so a CTA can cross a sequence boundary without a stall.
// Warp roles: 0 TMA producer, 1 MMA issuer (also allocates TMEM), 2..5 epilogue.
// In the prologue every warp counts the kept cold chunks of some sequences (the
// tile list is built from those counts; CTA 0 also writes them for the top-k).
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace li2 {

using namespace sm100;

constexpr int THREADS = 192;
constexpr int STAGES = 3;
constexpr int MAX_H = 128, MAX_D = 128;

struct __align__(1024) Smem {
    uint8_t keys[STAGES][MAX_D / 64][128 * 128];   // [atom][128 token rows][128 B]
    uint8_t q[2][MAX_D / 64][MAX_H * 128];          // [buffer][atom][H rows][128 B]
    uint64_t k_full[STAGES], k_empty[STAGES];
    uint64_t q_full[2], q_empty[2];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t mma_done;
    float w[MAX_H];                                 // head weights of the epilogue's current sequence
    uint32_t tmem_base;
    int abort_flag;
    // drain bookkeeping: last tile / query load issued into each slot (-1: none), and how
    // many of them the MMA issuer saw land
    int k_last[STAGES], q_last[2];
    int k_consumed, q_consumed;
    uint64_t never;                                 // no arrival ever: the failure-path test's wait
};

struct Params {
    const uint16_t *w_li;
    const int32_t *table;
    const int32_t *kept_idx;
    const int32_t *kept_count;
    const int32_t *window_start;
    int32_t *cold;                // out: kept chunks before the window, per sequence (written by CTA 0)
    float *scores;
    int32_t *status;
    int64_t n_slots;
    int B, H, D, table_stride, kept_cap;
    int stall;                    // failure-path test: the first wait waits on a barrier nothing arrives on
    // optional append of the decoded token (one epilogue warp of CTA b, b < B): its KV row
    // and indexer key go to position window_start[b] + window_len[b], then window_len[b] += 1
    const uint16_t *new_kv, *new_li;
    uint16_t *kv_pool, *li_pool;
    int64_t kv_stride;
    int kv_width;
    int32_t *window_len;
};

// The append of the decoded token, folded into the indexer launch: this kernel reads neither
// the window's rows nor window_len, so one warp of CTA b writes sequence b's new rows and
// advances its window while the pipeline fills; the attention launches that follow read them.
__device__ void append_token(const Params &p, int b, int lane) {
    int64_t row = -1;
    if (lane == 0) {
        const int pos = p.window_start[b] + p.window_len[b];
        const int chunk = pos / LSA_CHUNK;
        const int slot = (pos >= 0 && chunk < p.table_stride) ? p.table[(size_t)b * p.table_stride + chunk] : -1;
        row = (slot >= 0 && slot < p.n_slots) ? (int64_t)slot * LSA_CHUNK + pos % LSA_CHUNK : -1;
        if (row < 0) flag(p.status, LSA_DEV_TABLE);
    }
    row = __shfl_sync(0xffffffffu, row, 0);
    if (row >= 0) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.new_kv + (size_t)b * p.kv_width);
        uint4 *dst = reinterpret_cast<uint4 *>(p.kv_pool + row * p.kv_stride);
        for (int c = lane; c < p.kv_width / 8; c += 32) dst[c] = src[c];
        const uint4 *lsrc = reinterpret_cast<const uint4 *>(p.new_li + (size_t)b * p.D);
        uint4 *ldst = reinterpret_cast<uint4 *>(p.li_pool + row * p.D);
        for (int c = lane; c < p.D / 8; c += 32) ldst[c] = lsrc[c];
    }
    __syncwarp();
    if (lane == 0 && row >= 0) p.window_len[b] += 1;
}

// Starts fetching a tensor map (a __grid_constant__ parameter) so that the first copy through
// it does not wait for the descriptor.
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(map) : "memory");
}

// 1-CTA MMA and commit
__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(uint32_t(acc)));
}
__device__ __forceinline__ void commit(const uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tma_load_2d_local(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
            smem_addr(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}

// Work list shared by all roles of a CTA: tile t of the whole batch -> (sequence, first kept index).
struct Work {
    int tile_off[65];   // prefix of tiles per sequence (B <= 64)
    int cold[64];
    int first, last;    // tile range of this CTA
};

// Every CTA counts, per sequence, the kept chunks that lie before the recent
// window (they hold the indexer's candidates).  The kept list is ascending, so the
// count is the rank of the window's first chunk in it: each half-warp takes one
// sequence, samples 16 evenly spaced entries (one round of loads), and counts
// inside the one block of entries that straddles the window start (a second
// round).  CTA 0 also writes the counts out for the top-k pass that follows.
__device__ void count_cold(const Params &p, Work &wk, int warp, int lane) {
    const int half = lane >> 4, hl = lane & 15;
    const unsigned hmask = half ? 0xffff0000u : 0x0000ffffu;
    for (int b0 = 2 * warp; b0 < p.B; b0 += 2 * (THREADS / 32)) {
        const int b = b0 + half;
        const bool act = b < p.B;
        int cnt = 0, fw = 0;
        const int32_t *kept = p.kept_idx + (size_t)(act ? b : 0) * p.kept_cap;
        if (act) {
            cnt = min(max(p.kept_count[b], 0), p.kept_cap);
            fw = p.window_start[b] / LSA_CHUNK;
        }
        // block i = entries [i step, (i + 1) step); lane i samples the block's last entry
        const int step = (cnt + 15) / 16;
        bool below = false;
        if (act && cnt > 0) below = kept[min(cnt - 1, (hl + 1) * step - 1)] < fw;
        const int full = __popc(__ballot_sync(0xffffffffu, below) & hmask);   // blocks wholly below
        const int base = full * step;
        int c = 0;
#pragma unroll 8
        for (int i = hl; i < step; i += 16) {
            const int q = base + i;
            if (act && q < cnt) c += kept[q] < fw;
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (act && hl == 0) {
            const int n = min(cnt, base + c);
            wk.cold[b] = n;
            if (blockIdx.x == 0) p.cold[b] = n;
        }
    }
}

__device__ void build_work(const Params &p, Work &wk) {
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int b = 0; b < p.B; ++b) {
            wk.tile_off[b] = acc;
            acc += (wk.cold[b] + 1) >> 1;
        }
        wk.tile_off[p.B] = acc;
        wk.first = (int)((int64_t)blockIdx.x * acc / gridDim.x);
        wk.last = (int)((int64_t)(blockIdx.x + 1) * acc / gridDim.x);
    }
}

__device__ __forceinline__ int tile_seq(const Work &wk, int B, int t) {
    int b = 0;
    while (b + 1 < B && wk.tile_off[b + 1] <= t) ++b;
    return b;
}

__device__ __forceinline__ bool bounded(Smem &sm, const uint64_t *bar, uint32_t parity, int32_t *status,
                                        uint64_t limit = WAIT_NS) {
    if (sm.abort_flag) return false;
    if (mbar_wait(bar, parity, limit, &sm.abort_flag)) return true;
    if (!sm.abort_flag) flag(status, LSA_DEV_TIMEOUT);
    sm.abort_flag = 1;
    return false;
}

__global__ void __launch_bounds__(THREADS, 1)
li_score_kernel(const __grid_constant__ CUtensorMap key_map, const __grid_constant__ CUtensorMap q_map,
                const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023));
    __shared__ Work wk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int atoms = p.D / 64;

    if (threadIdx.x == 32) {
        prefetch_tensormap(&key_map);
        prefetch_tensormap(&q_map);
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) { mbar_init(&sm.k_full[i], 1); mbar_init(&sm.k_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.q_full[i], 1); mbar_init(&sm.q_empty[i], 1);
            mbar_init(&sm.acc_full[i], 1); mbar_init(&sm.acc_empty[i], 1);
        }
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.never, 1);
        for (int i = 0; i < STAGES; ++i) sm.k_last[i] = -1;
        sm.q_last[0] = sm.q_last[1] = -1;
        sm.k_consumed = sm.q_consumed = 0;
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    count_cold(p, wk, warp, lane);
    if (warp == 1) asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                                    smem_addr(&sm.tmem_base)), "r"(256));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    build_work(p, wk);
    __syncthreads();
    const uint32_t tmem = sm.tmem_base;
    const int t0 = wk.first, t1 = wk.last;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        int kslot = 0;
        uint32_t kpar = 0;
        int cur_b = -1, qbuf = 1, qswitch = 0;
        // Pool slots of the chunks of 16 tiles are looked up at once, lane i holding
        // chunk i & 1 of tile base + i / 2 (the slot count means "zero fill"), and the
        // next 16 are in flight meanwhile, so the two dependent lookups per chunk
        // (kept list, then chunk table) stay off the path from one tile to the next.
        auto lookup = [&](int base) {
            const int tt = base + (lane >> 1), i = lane & 1;
            int slot = (int)p.n_slots;
            if (tt < t1) {
                const int bb = tile_seq(wk, p.B, tt);
                const int j = 2 * (tt - wk.tile_off[bb]) + i;
                if (j < wk.cold[bb]) {
                    const int chunk = p.kept_idx[(size_t)bb * p.kept_cap + j];
                    const int sl = (chunk >= 0 && chunk < p.table_stride) ? p.table[(size_t)bb * p.table_stride + chunk] : -1;
                    if (sl >= 0 && sl < p.n_slots) slot = sl;
                }
            }
            return slot;
        };
        int batch = t0, slots = lookup(t0), slots_next = lookup(t0 + 16);
        for (int t = t0; t < t1; ++t) {
            if (t - batch == 16) {
                batch += 16;
                slots = slots_next;
                slots_next = lookup(batch + 16);
            }
            const int s0 = __shfl_sync(0xffffffffu, slots, 2 * (t - batch)), s1 = __shfl_sync(0xffffffffu, slots, 2 * (t - batch) + 1);
            const int b = tile_seq(wk, p.B, t);
            if (b != cur_b) {                              // query heads and weights of a new sequence
                cur_b = b;
                qbuf ^= 1;
                if (qswitch >= 2 && !bounded(sm, &sm.q_empty[qbuf], ((qswitch - 2) >> 1) & 1, p.status)) break;
                ++qswitch;
                if (lane == 0) {
                    expect_tx(&sm.q_full[qbuf], (uint32_t)(atoms * p.H * 128));
                    for (int a = 0; a < atoms; ++a) tma_load_2d_local(sm.q[qbuf][a], &q_map, 64 * a, b * p.H, &sm.q_full[qbuf]);
                    sm.q_last[qbuf] = qswitch - 1;
                }
                __syncwarp();
            }
            if (!bounded(sm, &sm.k_empty[kslot], kpar ^ 1u, p.status)) break;
            if (lane == 0) {
                const int j0 = 2 * (t - wk.tile_off[b]);
                const int nck = min(2, wk.cold[b] - j0);
                expect_tx(&sm.k_full[kslot], (uint32_t)(nck * atoms * 64 * 128));
                for (int i = 0; i < nck; ++i) {
                    const int slot = i ? s1 : s0;   // out of range (no slot): zero fill
                    for (int a = 0; a < atoms; ++a)
                        tma_load_2d_local(sm.keys[kslot][a] + i * 64 * 128, &key_map, 64 * a, slot * LSA_CHUNK,
                                          &sm.k_full[kslot]);
                }
                sm.k_last[kslot] = t - t0;
            }
            __syncwarp();
            if (++kslot == STAGES) { kslot = 0; kpar ^= 1u; }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16_f32(128, p.H, false, false);
        int kslot = 0;
        uint32_t kpar = 0;
        int cur_b = -1, qbuf = 1, qswitch = 0;
        bool ok = true;
        if (p.stall) ok = bounded(sm, &sm.never, 0, p.status, TEST_STALL_NS);
        for (int t = t0, u = 0; t < t1 && ok; ++t, ++u) {
            const int b = tile_seq(wk, p.B, t);
            if (b != cur_b) {
                if (cur_b >= 0 && lane == 0) commit(&sm.q_empty[qbuf]);   // previous buffer free after its MMAs
                cur_b = b;
                qbuf ^= 1;
                ok = bounded(sm, &sm.q_full[qbuf], (qswitch >> 1) & 1, p.status);
                ++qswitch;
                if (!ok) break;
                if (lane == 0) sm.q_consumed = qswitch;
            }
            const int ab = u & 1;
            if (u >= 2 && !(ok = bounded(sm, &sm.acc_empty[ab], ((u - 2) >> 1) & 1, p.status))) break;
            if (!(ok = bounded(sm, &sm.k_full[kslot], kpar, p.status))) break;
            if (lane == 0) sm.k_consumed = u + 1;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t d = tmem + 64 * ab * (p.H > 64 ? 2 : 1);
                for (int a = 0; a < atoms; ++a) {
                    const uint64_t ad = smem_desc_sw128(smem_addr(sm.keys[kslot][a]), 16, 1024);
                    const uint64_t bd = smem_desc_sw128(smem_addr(sm.q[qbuf][a]), 16, 1024);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) umma(d, ad + 2 * k4, bd + 2 * k4, idesc, (a | k4) != 0);
                }
                commit(&sm.k_empty[kslot]);
                commit(&sm.acc_full[ab]);
            }
            __syncwarp();
            if (++kslot == STAGES) { kslot = 0; kpar ^= 1u; }
        }
        if (cur_b >= 0 && lane == 0) commit(&sm.q_empty[qbuf]);
        if (lane == 0) {                                   // every MMA has completed before TMEM is released
            commit(&sm.mma_done);
            if (!mbar_wait(&sm.mma_done, 0, WAIT_NS)) flag(p.status, LSA_DEV_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue: one token row per thread
        if (warp == 2 && p.new_kv && (int)blockIdx.x < p.B) append_token(p, blockIdx.x, lane);
        const int L = threadIdx.x - 64;                       // 0..127
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const int row = 32 * (warp & 3) + lane;               // TMEM lane = token row of the tile
        bool ok = true;
        int w_b = -1;
        for (int t = t0, u = 0; t < t1; ++t, ++u) {
            const int b = tile_seq(wk, p.B, t);
            if (b != w_b) {   // head weights of a new sequence into shared memory
                named_barrier(1, 128);   // the previous weights are no longer read
                for (int h = L; h < p.H; h += 128) sm.w[h] = bf16_to_f32(p.w_li[(size_t)b * p.H + h]);
                named_barrier(1, 128);
                w_b = b;
            }
            // the row's chunk and slot are looked up while the MMA runs
            const int j0 = 2 * (t - wk.tile_off[b]);
            const int jj = j0 + (row >> 6);
            int slot = -1;
            if (jj < wk.cold[b]) {
                const int chunk = p.kept_idx[(size_t)b * p.kept_cap + jj];
                slot = (chunk >= 0 && chunk < p.table_stride) ? p.table[(size_t)b * p.table_stride + chunk] : -1;
            }
            const int ab = u & 1;
            if (ok) ok = bounded(sm, &sm.acc_full[ab], (u >> 1) & 1, p.status);
            tc_fence_after();
            const uint32_t base = tmem + lane_base + 64 * ab * (p.H > 64 ? 2 : 1);
            float acc = 0.f;
            for (int c0 = 0; c0 < p.H; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(base + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) acc += sm.w[c0 + i] * fmaxf(__uint_as_float(v[i]), 0.f);
            }
            tc_fence_before();
            named_barrier(1, 128);
            if (L == 0) arrive(&sm.acc_empty[ab]);
            // write the score of this row if it belongs to a kept cold chunk of the sequence
            if (ok && jj < wk.cold[b]) {
                const bool valid = slot >= 0 && slot < p.n_slots;
                if (!valid && (row & 63) == 0) flag(p.status, LSA_DEV_TABLE);
                p.scores[((size_t)b * p.kept_cap + jj) * LSA_CHUNK + (row & 63)] = valid ? acc : -INFINITY;
            }
        }
    }
    __syncthreads();
    if (sm.abort_flag) {
        // After an abort every TMA load issued lands before the CTA leaves: per key slot
        // and query buffer the last load whose full phase the MMA issuer did not see.
        if (threadIdx.x == 0) {
            for (int i = 0; i < STAGES; ++i)
                if (sm.k_last[i] >= sm.k_consumed)
                    (void)mbar_wait(&sm.k_full[i], (uint32_t)(sm.k_last[i] / STAGES) & 1u, WAIT_NS);
            for (int j = 0; j < 2; ++j)
                if (sm.q_last[j] >= sm.q_consumed)
                    (void)mbar_wait(&sm.q_full[j], (uint32_t)(sm.q_last[j] >> 1) & 1u, WAIT_NS);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(256));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
}

// --------------------------------------------------------------- host side --

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

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

bool shape_ok(int H, int D, int B) { return (H == 32 || H == 64 || H == 128) && (D == 64 || D == 128) && B <= 64; }

int launch(const uint16_t *q_li, const uint16_t *w_li, const uint16_t *li_pool, int64_t n_slots, const int32_t *table,
           int table_stride, const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
           const int32_t *window_start, int32_t *cold, int B, int H, int D, float *scores, int32_t *status,
           cudaStream_t stream, const AppendArgs *app) {
    CUtensorMap key_map, q_map;
    if (!make_map(&key_map, li_pool, D, (uint64_t)n_slots * LSA_CHUNK, LSA_CHUNK))
        return fail(LSA_ERR_CUDA, "lsa_topk: cuTensorMapEncodeTiled failed for the indexer key pool");
    if (!make_map(&q_map, q_li, D, (uint64_t)B * H, H))
        return fail(LSA_ERR_CUDA, "lsa_topk: cuTensorMapEncodeTiled failed for the indexer queries");
    Params prm;
    prm.w_li = w_li; prm.table = table; prm.kept_idx = kept_idx; prm.kept_count = kept_count;
    prm.window_start = window_start; prm.cold = cold; prm.scores = scores; prm.status = status; prm.n_slots = n_slots;
    prm.B = B; prm.H = H; prm.D = D; prm.table_stride = table_stride; prm.kept_cap = kept_cap;
    prm.stall = take_test_stall(LSA_TEST_STALL_INDEXER);
    prm.new_kv = app ? app->new_kv : nullptr;
    prm.new_li = app ? app->new_li : nullptr;
    prm.kv_pool = app ? app->kv_pool : nullptr;
    prm.li_pool = app ? app->li_pool : nullptr;
    prm.kv_stride = app ? app->kv_stride : 0;
    prm.kv_width = app ? app->kv_width : 0;
    prm.window_len = app ? app->window_len : nullptr;
    const size_t smem = sizeof(Smem) + 1024;
    LSA_CUDA(cudaFuncSetAttribute(li_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    li_score_kernel<<<sm_count(), THREADS, smem, stream>>>(key_map, q_map, prm);
    return check_launch("li_score_kernel (sm100)");
}

}  // namespace li2
}  // namespace lsa
