// sparse_decode_sm100.cu -- a4 on 5th-generation tensor cores: latent (MLA)
// sparse decode attention for 128 query heads over 576-wide KV rows (V = the
// first 512 columns), top-k rows plus the recent window.
// (arXiv 2606.09079: core attention over the selected entries and the most
// recent 8000 tokens, cjcn.com.cn article section 2; gist.science explainer 2.1.)
//
// A cluster of two CTAs (two SMs) owns one (sequence, split).  Every MMA is a
// cta_group::2 tcgen05.mma with M = 128 query heads: CTA r holds heads
// 64r..64r+63 of Q and of P in its shared memory, the B operand is split by
// N between the pair, and each CTA's tensor memory receives its own heads'
// rows of the result.
//   S = Q K^T   N = 64 kv rows per tile (each CTA loads 32 rows x 576 columns)
//   O += P V    N = 256 value columns per MMA, two MMAs per tile (each CTA
//               loads all 64 rows x its 2 x 128 value columns)
// TMEM per CTA: two S buffers of 32 columns and O = 64 heads x 512 values in
// 256 columns.  Rows are gathered by TMA tile::gather4 (4 rows per load,
// 128-byte swizzle) through the chunk table.  Warp roles:
//   0  K producer + tile-validity masks      1  V producer
//   2  MMA issuer (even CTA only)            3  TMEM allocator
//   4..7  softmax, O rescale, epilogue (one thread per TMEM lane)
// The online softmax is evaluated in the log2 domain; the reference maximum
// is only moved when a row maximum grows by more than 2^8, which keeps P <= 256
// in bf16 and makes O rescales rare.  Every mbarrier wait is bounded: on
// timeout the kernel sets LSA_DEV_TIMEOUT, drains and exits.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace mla2 {

using namespace sm100;

constexpr int HPC = 64;           // heads per CTA
constexpr int HQ = 128;           // heads per cluster
constexpr int DQK = 576, DV = 512;
constexpr int NTILE = 64;         // kv rows per tile
constexpr int KCH = DQK / 64;     // 9 column chunks of 64
constexpr int KST = 16;           // K ring: [32 rows x 64 cols] stages
constexpr int VST = 4;            // V ring: [2 atoms][64 rows][64 cols] stages
constexpr int INFO = 4;           // tile-validity ring
constexpr int THREADS = 256;
constexpr float RESCALE_LOG2 = 8.f;
constexpr uint32_t WAIT_LIMIT = 1u << 22;   // polls before a wait gives up (~seconds)

// TMEM columns
constexpr uint32_t TM_S = 0;      // S buffers at 0 and 32
constexpr uint32_t TM_O = 64;     // O at 64..319
constexpr uint32_t TM_COLS = 512;

struct __align__(1024) Smem {
    uint8_t q[KCH][HPC * 128];          // 9 x [64 heads][128 B], 128B-swizzled, K-major
    uint8_t k[KST][32 * 128];           // [32 kv rows][64 cols]
    uint8_t v[VST][2][NTILE * 128];     // [value atom][64 kv rows][64 value cols], MN-major
    uint8_t p[2][HPC * 128];            // [64 heads][64 kv], K-major
    uint64_t k_full[KST], k_empty[KST];
    uint64_t v_full[VST], v_empty[VST];
    uint64_t q_full;
    uint64_t s_full[2], s_empty[2], p_full[2];
    uint64_t pv_done[2], mma_done;   // pv_done[s]: P.V of the tiles using P buffer s
    uint64_t info_full[INFO], info_empty[INFO];
    unsigned long long info_mask[INFO];
    float red[128];
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const int32_t *table;
    const int32_t *topk_idx;
    const int32_t *topk_count;
    const int32_t *window_start;
    const int32_t *window_len;
    float *o_part, *m_part, *l_part;
    int32_t *status;
    int64_t n_rows_pool;   // n_slots * 64
    int table_stride, k, n_splits;
    float scale_log2;
};

// Tiles of one sequence: ceil(tk/64) top-k tiles, then the window chunk by chunk.
struct SeqTiles {
    int tk, wstart, wlen, t_topk, total;
    __device__ SeqTiles(const Params &p, int b) {
        tk = min(max(p.topk_count[b], 0), p.k);
        wstart = p.window_start[b];
        wlen = max(p.window_len[b], 0);
        t_topk = (tk + NTILE - 1) / NTILE;
        total = t_topk + (wlen + NTILE - 1) / NTILE;
    }
    // Window tile t (t >= t_topk) covers one whole chunk slot: first pool row of
    // the slot (-2 if the chunk has no slot) and the number of valid rows.
    __device__ int64_t window_slot_row(const Params &p, int b, int t, int *n_valid) const {
        const int j = t - t_topk;
        *n_valid = min(NTILE, wlen - NTILE * j);
        const int chunk = (wstart >> 6) + j;
        if (wstart < 0 || chunk >= p.table_stride) return -2;
        const int slot = p.table[(size_t)b * p.table_stride + chunk];
        const int64_t g = (int64_t)slot * LSA_CHUNK;
        if (slot < 0 || g >= p.n_rows_pool) return -2;
        return g;
    }
    // Global pool row of row i (0..63) of tile t, or -1.
    __device__ int64_t row(const Params &p, int b, int t, int i) const {
        int pos;
        if (t < t_topk) {
            const int r = t * NTILE + i;
            if (r >= tk) return -1;
            pos = p.topk_idx[(size_t)b * p.k + r];
        } else {
            const int r = (t - t_topk) * NTILE + i;
            if (r >= wlen) return -1;
            pos = wstart + r;
        }
        if (pos < 0) return -2;
        const int chunk = pos >> 6;
        if (chunk >= p.table_stride) return -2;
        const int slot = p.table[(size_t)b * p.table_stride + chunk];
        const int64_t g = (int64_t)slot * LSA_CHUNK + (pos & 63);
        if (slot < 0 || g >= p.n_rows_pool) return -2;
        return g;
    }
};

__device__ __forceinline__ void set_abort(Smem &sm, int32_t *status) {
    sm.abort_flag = 1;
    flag(status, LSA_DEV_TIMEOUT);
}

// Warp-uniform bounded wait (lane 0 polls, result broadcast).
__device__ __forceinline__ bool warp_wait(Smem &sm, const uint64_t *bar, uint32_t parity, int32_t *status) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        ok = sm.abort_flag == 0 && mbar_wait(bar, parity, WAIT_LIMIT);
        if (!ok) set_abort(sm, status);
    }
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__global__ void __launch_bounds__(THREADS, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap kv_map32,
                  const __grid_constant__ CUtensorMap kv_map64, const __grid_constant__ CUtensorMap q_map,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int split = blockIdx.x >> 1, b = blockIdx.y;

    if (threadIdx.x == 0) {
        for (int i = 0; i < KST; ++i) { mbar_init(&sm.k_full[i], 2); mbar_init(&sm.k_empty[i], 1); }
        for (int i = 0; i < VST; ++i) { mbar_init(&sm.v_full[i], 2); mbar_init(&sm.v_empty[i], 1); }
        mbar_init(&sm.q_full, 2);
        for (int i = 0; i < 2; ++i) { mbar_init(&sm.s_full[i], 1); mbar_init(&sm.s_empty[i], 2); mbar_init(&sm.p_full[i], 2); }
        mbar_init(&sm.pv_done[0], 1);
        mbar_init(&sm.pv_done[1], 1);
        mbar_init(&sm.mma_done, 1);
        for (int i = 0; i < INFO; ++i) { mbar_init(&sm.info_full[i], 1); mbar_init(&sm.info_empty[i], 1); }
        sm.abort_flag = 0;
        fence_mbar_init_cluster();
    }
    if (warp == 3) tmem_alloc_pair(&sm.tmem_base, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();
    const uint32_t tmem = sm.tmem_base;

    const SeqTiles st(p, b);
    // Tiles are dealt round-robin: split s takes tiles s, s + n_splits, ...  The
    // gathered top-k tiles (first in the tile list, and dearer to load than the
    // chunk-aligned window tiles) are thereby spread evenly over the splits.
    const int n_tiles = split < st.total ? (st.total - 1 - split) / p.n_splits + 1 : 0;
    const int u0 = split, ustride = p.n_splits;

    if (warp == 0 && n_tiles > 0) {
        // ------------------------------------------------ K producer + Q
        if (lane == 0) {
            const uint32_t qf = map_to_rank(&sm.q_full, 0);
            mbar_arrive_expect_tx_cluster(qf, KCH * HPC * 128);
            for (int c = 0; c < KCH; ++c) tma_load_2d(sm.q[c], &q_map, 64 * c, b * HQ + HPC * (int)rank, qf);
        }
        uint32_t kc = 0;
        // row indices of the next top-k tile are loaded while the current tile is issued
        int64_t n0 = -1, n1 = -1;
        if (u0 < st.t_topk) { n0 = st.row(p, b, u0, lane); n1 = st.row(p, b, u0, lane + 32); }
        for (int u = 0; u < n_tiles; ++u) {
            const int t = u0 + u * ustride;
            const bool window = t >= st.t_topk;
            const int64_t g0 = n0, g1 = n1;
            if (u + 1 < n_tiles && t + ustride < st.t_topk) {
                n0 = st.row(p, b, t + ustride, lane);
                n1 = st.row(p, b, t + ustride, lane + 32);
            }
            unsigned long long mask;
            int64_t slot_row = -1;
            if (window) {
                int nv;
                slot_row = st.window_slot_row(p, b, t, &nv);
                if (slot_row == -2) flag(p.status, LSA_DEV_TABLE);
                mask = slot_row < 0 ? 0ull : (nv >= 64 ? ~0ull : ((1ull << nv) - 1ull));
            } else {
                if ((g0 == -2 || g1 == -2)) flag(p.status, LSA_DEV_TABLE);
                const unsigned lo = __ballot_sync(0xffffffffu, g0 >= 0), hi = __ballot_sync(0xffffffffu, g1 >= 0);
                mask = (unsigned long long)lo | ((unsigned long long)hi << 32);
            }
            if (!warp_wait(sm, &sm.info_empty[u % INFO], ((u / INFO) + 1) & 1, p.status)) break;
            if (lane == 0) {
                sm.info_mask[u % INFO] = mask;
                asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(&sm.info_full[u % INFO])) : "memory");
            }
            const int64_t mine = rank ? g1 : g0;
            const int gr = mine >= 0 ? (int)mine : (int)p.n_rows_pool;   // out of range -> zero fill
            const int r0 = __shfl_sync(0xffffffffu, gr, (4 * lane) & 31), r1 = __shfl_sync(0xffffffffu, gr, (4 * lane + 1) & 31);
            const int r2 = __shfl_sync(0xffffffffu, gr, (4 * lane + 2) & 31), r3 = __shfl_sync(0xffffffffu, gr, (4 * lane + 3) & 31);
            const int wy = slot_row >= 0 ? (int)slot_row + 32 * (int)rank : (int)p.n_rows_pool;
            bool ok = true;
            for (int c = 0; c < KCH; ++c, ++kc) {
                const int s = kc % KST;
                ok = warp_wait(sm, &sm.k_empty[s], ((kc / KST) + 1) & 1, p.status);
                if (!ok) break;
                const uint32_t full = map_to_rank(&sm.k_full[s], 0);
                if (lane == 0) {
                    mbar_arrive_expect_tx_cluster(full, 32 * 128);
                    if (window) tma_load_2d(sm.k[s], &kv_map32, 64 * c, wy, full);
                }
                __syncwarp();
                if (!window && lane < 8) tma_gather4(sm.k[s] + lane * 512, &kv_map, 64 * c, r0, r1, r2, r3, full);
            }
            if (!ok) break;
        }
    } else if (warp == 1 && n_tiles > 0) {
        // ------------------------------------------------ V producer
        uint32_t vc = 0;
        int64_t n0 = -1, n1 = -1;
        if (u0 < st.t_topk) { n0 = st.row(p, b, u0, lane); n1 = st.row(p, b, u0, lane + 32); }
        for (int u = 0; u < n_tiles; ++u) {
            const int t = u0 + u * ustride;
            const bool window = t >= st.t_topk;
            const int64_t g0 = n0, g1 = n1;
            if (u + 1 < n_tiles && t + ustride < st.t_topk) {
                n0 = st.row(p, b, t + ustride, lane);
                n1 = st.row(p, b, t + ustride, lane + 32);
            }
            int wy = (int)p.n_rows_pool;
            if (window) {
                int nv;
                const int64_t sr = st.window_slot_row(p, b, t, &nv);
                if (sr >= 0) wy = (int)sr;
            }
            const int a0 = g0 >= 0 ? (int)g0 : (int)p.n_rows_pool, a1 = g1 >= 0 ? (int)g1 : (int)p.n_rows_pool;
            // lane -> (value atom a = lane / 16, row group gq = lane % 16: rows 4gq .. 4gq + 3)
            const int gq = lane & 15, a = lane >> 4;
            int r[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 4 * gq + i;
                const int x0 = __shfl_sync(0xffffffffu, a0, row & 31), x1 = __shfl_sync(0xffffffffu, a1, row & 31);
                r[i] = row < 32 ? x0 : x1;
            }
            bool ok = true;
            for (int j = 0; j < 2 && ok; ++j, ++vc) {
                const int s = vc % VST;
                ok = warp_wait(sm, &sm.v_empty[s], ((vc / VST) + 1) & 1, p.status);
                if (!ok) break;
                const uint32_t full = map_to_rank(&sm.v_full[s], 0);
                const int col0 = 256 * j + 128 * (int)rank;
                if (lane == 0) {
                    mbar_arrive_expect_tx_cluster(full, 2 * NTILE * 128);
                    if (window) {
                        tma_load_2d(sm.v[s][0], &kv_map64, col0, wy, full);
                        tma_load_2d(sm.v[s][1], &kv_map64, col0 + 64, wy, full);
                    }
                }
                __syncwarp();
                if (!window) tma_gather4(sm.v[s][a] + gq * 512, &kv_map, col0 + 64 * a, r[0], r[1], r[2], r[3], full);
            }
            if (!ok) break;
        }
    } else if (warp == 2 && rank == 0 && n_tiles > 0) {
        // ------------------------------------------------ MMA issuer (even CTA)
        // Descriptors are built once; a byte offset o within shared memory is
        // o >> 4 added to the descriptor's start-address field.
        constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, NTILE, false, false);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);
        const uint64_t qd0 = smem_desc_sw128(smem_addr(sm.q[0]), 16, 1024);
        const uint64_t kd0 = smem_desc_sw128(smem_addr(sm.k[0]), 16, 1024);
        const uint64_t pd0 = smem_desc_sw128(smem_addr(sm.p[0]), 16, 1024);
        const uint64_t vd0 = smem_desc_sw128(smem_addr(sm.v[0][0]), NTILE * 128, 1024);
        constexpr uint64_t Q_CHUNK = (HPC * 128) >> 4, K_STAGE = (32 * 128) >> 4, P_BUF = (HPC * 128) >> 4;
        constexpr uint64_t V_STAGE = (2 * NTILE * 128) >> 4, K16 = 32 >> 4, V16 = (16 * 128) >> 4;
        bool ok = warp_wait(sm, &sm.q_full, 0, p.status);
        int kslot = 0, vslot = 0;
        uint32_t kpar = 0, vpar = 0;
        for (int u = -1; u < n_tiles && ok; ++u) {
            if (u + 1 < n_tiles) {                         // S(u+1) = Q K^T
                const int t = u + 1, sb = t & 1;
                ok = warp_wait(sm, &sm.s_empty[sb], ((t >> 1) + 1) & 1, p.status);
                tc_fence_after();
                const uint32_t d = tmem + TM_S + 32 * sb;
                for (int c = 0; c < KCH && ok; ++c) {
                    ok = warp_wait(sm, &sm.k_full[kslot], kpar, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint64_t a = qd0 + Q_CHUNK * c, bb = kd0 + K_STAGE * kslot;
                        umma_pair_ss(d, a, bb, IDESC_QK, c != 0);
                        umma_pair_ss(d, a + K16, bb + K16, IDESC_QK, true);
                        umma_pair_ss(d, a + 2 * K16, bb + 2 * K16, IDESC_QK, true);
                        umma_pair_ss(d, a + 3 * K16, bb + 3 * K16, IDESC_QK, true);
                        umma_commit_pair(&sm.k_empty[kslot], 0x3);
                    }
                    __syncwarp();
                    if (++kslot == KST) { kslot = 0; kpar ^= 1u; }
                }
                if (lane == 0) umma_commit_pair(&sm.s_full[sb], 0x3);
                __syncwarp();
            }
            if (u >= 0 && ok) {                            // O += P V for tile u
                const int sb = u & 1;
                ok = warp_wait(sm, &sm.p_full[sb], (u >> 1) & 1, p.status);
                tc_fence_after();
                const uint64_t a = pd0 + P_BUF * sb;
                for (int j = 0; j < 2 && ok; ++j) {
                    ok = warp_wait(sm, &sm.v_full[vslot], vpar, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint64_t bb = vd0 + V_STAGE * vslot;
                        const uint32_t d = tmem + TM_O + 128 * j;
                        umma_pair_ss(d, a, bb, IDESC_PV, u != 0);
                        umma_pair_ss(d, a + K16, bb + V16, IDESC_PV, true);
                        umma_pair_ss(d, a + 2 * K16, bb + 2 * V16, IDESC_PV, true);
                        umma_pair_ss(d, a + 3 * K16, bb + 3 * V16, IDESC_PV, true);
                        umma_commit_pair(&sm.v_empty[vslot], 0x3);
                    }
                    __syncwarp();
                    if (++vslot == VST) { vslot = 0; vpar ^= 1u; }
                }
                if (lane == 0) umma_commit_pair(&sm.pv_done[sb], 0x3);
                __syncwarp();
            }
        }
        if (lane == 0) umma_commit_pair(&sm.mma_done, 0x3);
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax + epilogue
        const int L = threadIdx.x - 128;        // TMEM lane of this thread
        const int h = L & 63, half = L >> 6;     // head within the CTA, kv half of the tile
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int u = 0; u < n_tiles; ++u) {
            const int s = u & 1;
            ok = ok && sm.abort_flag == 0;
            if (ok) ok = mbar_wait(&sm.info_full[u % INFO], (u / INFO) & 1, WAIT_LIMIT);
            const uint32_t vmask = ok ? (uint32_t)(sm.info_mask[u % INFO] >> (32 * half)) : 0u;
            if (ok) ok = mbar_wait(&sm.s_full[s], (u >> 1) & 1, WAIT_LIMIT);
            if (!ok && sm.abort_flag == 0) set_abort(sm, p.status);
            tc_fence_after();
            uint32_t raw[32];
            tmem_ld32(tmem + lane_base + TM_S + 32 * s, raw);
            tmem_wait_ld();
            tc_fence_before();
            named_barrier(1, 128);
            if (L == 0) {
                mbar_arrive_cluster(map_to_rank(&sm.s_empty[s], 0));
                asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(&sm.info_empty[u % INFO])) : "memory");
            }
            float sv[32];
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                sv[i] = (vmask >> i) & 1u ? __uint_as_float(raw[i]) * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, sv[i]);
            }
            sm.red[L] = mx;
            named_barrier(1, 128);
            mx = fmaxf(mx, sm.red[L ^ 64]);
            const float m_new = fmaxf(m_run, mx);
            m_run = m_new;
            // P buffer s is free once P.V of tile u-2 completed.  O must be stable
            // (P.V of tile u-1 done) only when it is rescaled, which is rare.
            if (u > 1 && ok) {
                ok = mbar_wait(&sm.pv_done[s], ((u - 2) >> 1) & 1, WAIT_LIMIT);
                if (!ok && sm.abort_flag == 0) set_abort(sm, p.status);
            }
            if (m_new > -INFINITY && (m_ref == -INFINITY || m_new > m_ref + RESCALE_LOG2)) {
                const float alpha = m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_new);
                if (u > 0) {
                    if (ok) {
                        ok = mbar_wait(&sm.pv_done[(u - 1) & 1], ((u - 1) >> 1) & 1, WAIT_LIMIT);
                        if (!ok && sm.abort_flag == 0) set_abort(sm, p.status);
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int q = 0; q < 8; ++q) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + TM_O + 32 * q, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(tmem + lane_base + TM_O + 32 * q, o);
                    }
                    tmem_wait_st();
                }
                l *= alpha;
                m_ref = m_new;
            }
            float psum = 0.f;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = exp2f(sv[2 * i] - m_ref), p1 = exp2f(sv[2 * i + 1] - m_ref);
                const float q0 = m_ref == -INFINITY ? 0.f : p0, q1 = m_ref == -INFINITY ? 0.f : p1;
                psum += q0 + q1;
                pk[i] = pack_bf16x2(q0, q1);
            }
            l += psum;
            uint8_t *prow = sm.p[s] + h * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int chunk = 4 * half + c;
                *reinterpret_cast<uint4 *>(prow + ((chunk ^ (h & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_barrier(1, 128);
            if (L == 0) mbar_arrive_cluster(map_to_rank(&sm.p_full[s], 0));
        }
        // ---- epilogue: wait for the last P.V, then write the partial
        if (n_tiles > 0 && ok) {
            ok = mbar_wait(&sm.pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, WAIT_LIMIT);
            if (!ok && sm.abort_flag == 0) set_abort(sm, p.status);
        }
        tc_fence_after();
        sm.red[L] = l;
        named_barrier(1, 128);
        const float l_tot = l + sm.red[L ^ 64];
        const int head = HPC * (int)rank + h;
        const size_t part = ((size_t)b * p.n_splits + split) * HQ + head;
        if (half == 0) {
            p.m_part[part] = n_tiles > 0 ? m_ref : -INFINITY;
            p.l_part[part] = n_tiles > 0 ? l_tot : 0.f;
        }
        float *orow = p.o_part + part * DV;
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {
            uint32_t o[32];
            if (n_tiles > 0) {
                tmem_ld32(tmem + lane_base + TM_O + 32 * q, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
            // O columns 0..127 hold values 0..255 split by lane half; 128..255 hold 256..511
            const int j = q >> 2, within = (q & 3) * 32;
            float4 *dst = reinterpret_cast<float4 *>(orow + 256 * j + 128 * half + within);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                     __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
        tc_fence_before();
    }

    // ---- teardown: every MMA finished before TMEM is released; no CTA leaves early
    if (warp == 3 && n_tiles > 0) {
        // the even CTA's MMA thread commits mma_done to both CTAs after its last MMA
        if (lane == 0 && !mbar_wait(&sm.mma_done, 0, WAIT_LIMIT)) set_abort(sm, p.status);
        __syncwarp();
    }
    __syncthreads();
    if (sm.abort_flag) __nanosleep(20000);   // let in-flight TMA loads land before the CTA exits
    cluster_sync();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TM_COLS);
        tmem_relinquish_pair();
    }
}

// --------------------------------------------------------------- host side --

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encoder() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    }
    return fn;
}

static bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                     uint32_t box_cols, uint32_t box_rows) {
    EncodeTiled enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t smem_bytes() { return sizeof(Smem) + 1024; }

int max_splits(int B) {
    const int clusters = sm_count() / 2;
    return max(1, clusters / max(B, 1));
}

int launch(const uint16_t *q, const uint16_t *kv_pool, int64_t k_stride, int64_t n_slots, const int32_t *table,
           int table_stride, const int32_t *topk_idx, const int32_t *topk_count, int k, const int32_t *window_start,
           const int32_t *window_len, int B, float scale, int n_splits, float *o_part, float *m_part, float *l_part,
           int32_t *status, cudaStream_t stream) {
    CUtensorMap kv_map, kv_map32, kv_map64, q_map;
    const uint64_t pool_rows = (uint64_t)n_slots * LSA_CHUNK;
    if (!make_map(&kv_map, kv_pool, DQK, pool_rows, (uint64_t)k_stride * 2, 64, 1) ||
        !make_map(&kv_map32, kv_pool, DQK, pool_rows, (uint64_t)k_stride * 2, 64, 32) ||
        !make_map(&kv_map64, kv_pool, DQK, pool_rows, (uint64_t)k_stride * 2, 64, 64))
        return fail(LSA_ERR_CUDA, "lsa_sparse_decode: cuTensorMapEncodeTiled failed for the KV pool");
    if (!make_map(&q_map, q, DQK, (uint64_t)B * HQ, DQK * 2, 64, 64))
        return fail(LSA_ERR_CUDA, "lsa_sparse_decode: cuTensorMapEncodeTiled failed for q");
    Params prm;
    prm.table = table; prm.topk_idx = topk_idx; prm.topk_count = topk_count;
    prm.window_start = window_start; prm.window_len = window_len;
    prm.o_part = o_part; prm.m_part = m_part; prm.l_part = l_part; prm.status = status;
    prm.n_rows_pool = n_slots * LSA_CHUNK; prm.table_stride = table_stride; prm.k = k; prm.n_splits = n_splits;
    prm.scale_log2 = scale * 1.4426950408889634f;
    const size_t smem = smem_bytes();
    LSA_CUDA(cudaFuncSetAttribute(mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * n_splits, B, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LSA_CUDA(cudaLaunchKernelEx(&cfg, mla_decode_kernel, kv_map, kv_map32, kv_map64, q_map, prm));
    return LSA_OK;
}

}  // namespace mla2
}  // namespace lsa
