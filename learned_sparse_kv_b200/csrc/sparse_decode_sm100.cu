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
//   S = Q K^T   N = 64 kv rows per tile (CTA r holds rows 32r..32r+31, all 576 columns)
//   O += P V    N = 256 value columns per MMA (CTA r holds all 64 rows of value
//               columns 128r..128r+127 and 256+128r..); P is passed as the sum
//               of two bf16 parts, hi = bf16(P) and lo = bf16(P - hi), so every
//               K step takes four MMAs and P keeps ~16 bits of precision
// TMEM per CTA: two S buffers of 32 columns and O = 64 heads x 512 values in
// 256 columns.
//
// Loading a tile is one operation per operand: a 3D TMA box {64 columns, 32
// rows, 9 column chunks} fetches a CTA's K rows (36 KB) and a 4D box {64, 64
// rows, 2, 2} its value columns (32 KB), both straight into the 128-byte-swizzled
// operand layout.  Window tiles that are a whole aligned chunk slot are read
// from the pool; the other tiles (top-k rows, and window tiles that are not a
// whole aligned chunk) are first copied, 64 rows at a time, by stage_kernel
// into a contiguous staging buffer (missing rows zero-filled), so that they are
// TMA boxes too: that copy runs on every multiprocessor at the memory's rate,
// where row gathers inside this kernel were bound by the copies one
// multiprocessor keeps in flight and stalled the two-stage pipeline.  Two
// stages of each operand are in flight.
// Warp roles:
//   0      K producer (TMA), tile-validity masks
//   1      S = Q K^T issuer (even CTA)        2   O += P V issuer (even CTA)
//   3      TMEM allocator, V producer (TMA)
//   4..7   softmax, O rescale, epilogue (one thread per TMEM lane)
// The online softmax is evaluated in the log2 domain; the reference maximum
// is only moved when a row maximum grows by more than 2^8, which keeps P <= 256
// in bf16 and makes O rescales rare.  Every mbarrier wait is bounded: on
// timeout the kernel sets LSA_DEV_TIMEOUT and the abort flag of both CTAs, the
// other waits return, the tensor-core work issued so far completes, the even CTA
// waits for every TMA load still in flight, and the pair exits.
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
constexpr int STAGES = 2;         // tiles in flight per operand
constexpr int INFO = 4;           // tile-validity ring
constexpr int THREADS = 256;
constexpr uint32_t Q_BYTES = KCH * HPC * 128;          // per CTA
constexpr uint32_t K_BYTES = KCH * 32 * 128;           // per CTA and tile
constexpr uint32_t V_BYTES = 2 * 2 * NTILE * 128;      // per CTA and tile
constexpr float RESCALE_LOG2 = 8.f;

// TMEM columns
constexpr uint32_t TM_S = 0;      // S buffers at 0 and 32
constexpr uint32_t TM_O = 64;     // O at 64..319
constexpr uint32_t TM_COLS = 512;

struct __align__(1024) Smem {
    uint8_t q[KCH][HPC * 128];                 // 9 x [64 heads][128 B], 128B-swizzled, K-major
    uint8_t k[STAGES][KCH][32 * 128];          // [chunk][32 kv rows][64 cols]
    uint8_t v[STAGES][2][2][NTILE * 128];      // [value block j][atom][64 kv rows][64 value cols], MN-major
    uint8_t p[2][HPC * 128];                   // P = hi + lo: [part][64 heads][64 kv], K-major
    uint64_t k_full[STAGES], k_empty[STAGES];
    uint64_t v_full[STAGES], v_empty[STAGES];
    uint64_t q_full;
    uint64_t s_full[2], s_empty[2], p_full[2];
    uint64_t pv_done[2], mma_done;   // pv_done[u & 1]: P.V of tile u
    uint64_t info_full[INFO], info_empty[INFO];
    unsigned long long info_mask[INFO];
    float red[128];
    uint32_t tmem_base;
    int abort_flag;
    // drain bookkeeping: the tile of the last TMA load this CTA issued into each stage
    // (-1: none), and (even CTA) the tiles whose K / V full phase an issuer saw complete
    int last_k_tma[STAGES], last_v_tma[STAGES];
    int k_consumed, v_consumed, q_seen;
    uint64_t never;                  // no arrival ever: the failure-path test's wait
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA");

struct Params {
    const int32_t *table;
    const int32_t *topk_idx;
    const int32_t *topk_count;
    const int32_t *window_start;
    const int32_t *window_len;
    const uint8_t *pool;       // KV pool base (bytes)
    int64_t row_bytes;         // pool row stride in bytes
    float *o_part, *m_part, *l_part;
    int32_t *status;
    int64_t n_rows_pool;   // n_slots * 64
    int table_stride, k, n_splits;
    int stage_tiles;       // staging slots per sequence
    uint16_t *stage_mask;  // [B][stage_tiles][4]: valid rows of each staged tile, 16 per piece
    float scale_log2;
    int stall;             // failure-path test: the first wait waits on a barrier nothing arrives on
};

// Tiles of one sequence: ceil(tk/64) top-k tiles, then the window chunk by chunk.
struct SeqTiles {
    int tk, wstart, wlen, t_topk, total;
    bool aligned;
    __device__ SeqTiles(const Params &p, int b) {
        tk = min(max(p.topk_count[b], 0), p.k);
        wstart = p.window_start[b];
        wlen = max(p.window_len[b], 0);
        t_topk = (tk + NTILE - 1) / NTILE;
        total = t_topk + (wlen + NTILE - 1) / NTILE;
        aligned = (wstart & (NTILE - 1)) == 0;
    }
    // Top-k tiles, and window tiles that are not one whole chunk slot, are gathered row by row.
    __device__ bool gathered(int t) const {
        if (t < t_topk) return true;
        return !aligned || wlen - NTILE * (t - t_topk) < NTILE;
    }
    // Window tile t (t >= t_topk, aligned window) covers one whole chunk slot:
    // its first pool row, or -2 if the chunk has no slot.
    __device__ int64_t window_slot_row(const Params &p, int b, int t) const {
        const int chunk = (wstart >> 6) + (t - t_topk);
        if (wstart < 0 || chunk >= p.table_stride) return -2;
        const int slot = p.table[(size_t)b * p.table_stride + chunk];
        const int64_t g = (int64_t)slot * LSA_CHUNK;
        if (slot < 0 || g >= p.n_rows_pool) return -2;
        return g;
    }
    // Staging slot of gathered tile t: top-k tiles first, then (aligned window) the
    // last, partial window tile, or (unaligned window) every window tile in order.
    __device__ int stage_index(int t) const { return t < t_topk ? t : (aligned ? t_topk : t); }
    // Inverse: the gathered tile staged in slot g, or -1.
    __device__ int staged_tile(int g) const {
        if (g < t_topk) return g;
        if (aligned) return (g == t_topk && total > t_topk && gathered(total - 1)) ? total - 1 : -1;
        return g < total ? g : -1;
    }
    // Global pool row of row i (0..63) of tile t, -1 past the end of the row set, -2 if unmapped.
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

// Sets the abort flag of both CTAs of the pair (the peer's through distributed
// shared memory), so that every bounded wait of the pair returns at once.
__device__ __noinline__ void set_abort(Smem &sm, int32_t *status) {
    sm.abort_flag = 1;
    asm volatile("st.shared::cluster.s32 [%0], %1;\n" ::"r"(map_to_rank(&sm.abort_flag, cluster_rank() ^ 1u)), "r"(1)
                 : "memory");
    flag(status, LSA_DEV_TIMEOUT);
}

__device__ __forceinline__ int ld_peer_s32(const void *p) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];\n" : "=r"(v) : "r"(map_to_rank(p, cluster_rank() ^ 1u)) : "memory");
    return v;
}

// Warp-uniform bounded wait (lane 0 polls, result broadcast).
__device__ __forceinline__ bool warp_wait(Smem &sm, const uint64_t *bar, uint32_t parity, int32_t *status,
                                          uint64_t limit = WAIT_NS) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        ok = sm.abort_flag == 0 && mbar_wait(bar, parity, limit, &sm.abort_flag);
        if (!ok && sm.abort_flag == 0) set_abort(sm, status);
    }
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Same, acquiring at cluster scope (phases that the peer CTA's generic stores complete).
__device__ __forceinline__ bool warp_wait_cluster(Smem &sm, const uint64_t *bar, uint32_t parity, int32_t *status) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        ok = sm.abort_flag == 0 && mbar_wait_cluster(bar, parity, WAIT_NS, &sm.abort_flag);
        if (!ok && sm.abort_flag == 0) set_abort(sm, status);
    }
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Waits until the TMA load of the last tile issued into a stage has landed, if no issuer
// saw its full phase complete.  u0 / u1: that tile as issued by the even / odd CTA.
__device__ __forceinline__ void drain_stage(uint64_t *full, int u0, int u1, int consumed) {
    const int u = max(u0, u1);
    if (u < consumed) return;            // completed and consumed, or nothing issued (u = -1)
    if (u0 != u) mbar_arrive_local(full);   // the even CTA did not issue tile u
    if (u1 != u) mbar_arrive_local(full);   // the odd CTA did not issue tile u
    (void)mbar_wait(full, (uint32_t)(u >> 1) & 1u, WAIT_NS);
}

// grid (4 * stage_tiles, B), 128 threads: CTA (4 g + q, b) copies rows 16 q .. 16 q + 15
// of the gathered tile staged in slot g of sequence b (rows past the row set, or
// without a slot, as zeros) and writes which of them are valid into the tile's mask.  Each thread keeps its 9 loads of 16 bytes in flight
// before storing; a unit over four CTAs keeps four times the copies in flight of
// one CTA per unit.
constexpr int STAGE_ROWS = 16, STAGE_THREADS = 128;
__global__ void __launch_bounds__(STAGE_THREADS) stage_kernel(const Params p, uint8_t *__restrict__ stage) {
    constexpr int PIECES = DQK * 2 / 16;                              // 72 pieces of 16 bytes per row
    constexpr int PER_THREAD = STAGE_ROWS * PIECES / STAGE_THREADS;   // 9
    __shared__ int64_t rows[STAGE_ROWS];
    const int g = blockIdx.x >> 2, r0 = STAGE_ROWS * (blockIdx.x & 3), b = blockIdx.y;
    const SeqTiles st(p, b);
    const int t = st.staged_tile(g);
    if (t < 0) return;
    if (threadIdx.x < STAGE_ROWS) rows[threadIdx.x] = st.row(p, b, t, r0 + threadIdx.x);
    __syncthreads();
    if (threadIdx.x < 32) {
        // rows 16 q .. 16 q + 15 of the tile's validity mask (the attention's softmax reads it)
        const int64_t r = threadIdx.x < STAGE_ROWS ? rows[threadIdx.x] : -1;
        const unsigned valid = __ballot_sync(0xffffffffu, r >= 0), unmapped = __ballot_sync(0xffffffffu, r == -2);
        if (threadIdx.x == 0) {
            p.stage_mask[((size_t)b * p.stage_tiles + g) * 4 + (blockIdx.x & 3)] = (uint16_t)valid;
            if (unmapped) flag(p.status, LSA_DEV_TABLE);
        }
    }
    uint4 v[PER_THREAD];
#pragma unroll
    for (int i = 0; i < PER_THREAD; ++i) {
        const int q = threadIdx.x + STAGE_THREADS * i, r = q / PIECES, w = q - r * PIECES;
        const int64_t pr = rows[r];
        v[i] = pr >= 0 ? __ldg(reinterpret_cast<const uint4 *>(p.pool + pr * p.row_bytes) + w) : make_uint4(0, 0, 0, 0);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(stage + (((size_t)b * p.stage_tiles + g) * NTILE + r0) * (DQK * 2));
#pragma unroll
    for (int i = 0; i < PER_THREAD; ++i) dst[threadIdx.x + STAGE_THREADS * i] = v[i];
}

__global__ void __launch_bounds__(THREADS, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                  const __grid_constant__ CUtensorMap ks_map, const __grid_constant__ CUtensorMap vs_map,
                  const __grid_constant__ CUtensorMap q_map, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int split = blockIdx.x >> 1, b = blockIdx.y;
    // the sequence's row counts are read while the barriers and tensor memory are set up
    const SeqTiles st(p, b);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&sm.k_full[i], 2); mbar_init(&sm.k_empty[i], 1);
            mbar_init(&sm.v_full[i], 2); mbar_init(&sm.v_empty[i], 1);
        }
        mbar_init(&sm.q_full, 2);
        for (int i = 0; i < 2; ++i) { mbar_init(&sm.s_full[i], 1); mbar_init(&sm.s_empty[i], 2); mbar_init(&sm.p_full[i], 2); }
        mbar_init(&sm.pv_done[0], 1);
        mbar_init(&sm.pv_done[1], 1);
        mbar_init(&sm.mma_done, 2);   // one commit from each MMA issuer
        for (int i = 0; i < INFO; ++i) { mbar_init(&sm.info_full[i], 1); mbar_init(&sm.info_empty[i], 1); }
        mbar_init(&sm.never, 1);
        for (int i = 0; i < STAGES; ++i) sm.last_k_tma[i] = sm.last_v_tma[i] = -1;
        sm.k_consumed = sm.v_consumed = sm.q_seen = 0;
        sm.abort_flag = 0;
        fence_mbar_init_cluster();
    }
    if (warp == 3) tmem_alloc_pair(&sm.tmem_base, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();
    const uint32_t tmem = sm.tmem_base;

    // Tiles are dealt round-robin: split s takes tiles s, s + n_splits, ...  The
    // staged top-k tiles (first in the tile list) are thereby spread evenly over
    // the splits.  K (warp 0) and V (warp 3) have a producer each, so K of a later
    // tile never waits behind the P.V that frees a V stage.
    const int n_tiles = split < st.total ? (st.total - 1 - split) / p.n_splits + 1 : 0;
    const int u0 = split, ustride = p.n_splits;
    auto tile_of = [&](int u) { return u0 + u * ustride; };
    if ((warp == 0 || warp == 3) && n_tiles > 0) {
        // ------------------------------------------------ TMA producers (K + masks, V)
        const bool kprod = warp == 0;
        if (kprod && lane == 0) {
            const uint32_t qf = map_to_rank(&sm.q_full, 0);
            mbar_arrive_expect_tx_cluster(qf, Q_BYTES);
            tma_load_3d(sm.q[0], &q_map, 0, b * HQ + HPC * (int)rank, 0, qf);
        }
        auto locate = [&](int u, int64_t &slot_row) -> int {
            const int t = tile_of(u);
            if (st.gathered(t)) {
                slot_row = -2;
                return (b * p.stage_tiles + st.stage_index(t)) * NTILE;
            }
            slot_row = st.window_slot_row(p, b, t);
            return slot_row >= 0 ? (int)slot_row : (int)p.n_rows_pool;
        };
        int64_t sr0 = -2, sr1 = -2;
        int wy0 = locate(0, sr0), wy1 = n_tiles > 1 ? locate(1, sr1) : 0;
        for (int u = 0; u < n_tiles; ++u) {
            const int t = tile_of(u);
            const int s = u & 1;
            const uint32_t par = ((u >> 1) + 1) & 1;
            const int wy = s ? wy1 : wy0;
            const int64_t slot_row = s ? sr1 : sr0;
            const bool gath = st.gathered(t);
            if (kprod) {
                if (!warp_wait(sm, &sm.k_empty[s], par, p.status)) break;
                if (lane == 0) {
                    const uint32_t full = map_to_rank(&sm.k_full[s], 0);
                    mbar_arrive_expect_tx_cluster(full, K_BYTES);
                    tma_load_3d(sm.k[s][0], gath ? &ks_map : &k_map, 0, wy + 32 * (int)rank, 0, full);
                    sm.last_k_tma[s] = u;
                }
            } else {
                if (!warp_wait(sm, &sm.v_empty[s], par, p.status)) break;
                if (lane == 0) {
                    const uint32_t full = map_to_rank(&sm.v_full[s], 0);
                    mbar_arrive_expect_tx_cluster(full, V_BYTES);
                    tma_load_4d(sm.v[s][0][0], gath ? &vs_map : &v_map, 0, wy, 2 * (int)rank, 0, full);
                    sm.last_v_tma[s] = u;
                }
            }
            if (u + 2 < n_tiles) {
                if (s) wy1 = locate(u + 2, sr1);
                else wy0 = locate(u + 2, sr0);
            }
            if (kprod) {
                unsigned long long mask;
                if (!gath) {
                    if (slot_row == -2) flag(p.status, LSA_DEV_TABLE);
                    mask = slot_row < 0 ? 0ull : ~0ull;
                } else {
                    // written by the staging copy (which also flagged unmapped rows)
                    mask = *reinterpret_cast<const unsigned long long *>(
                        p.stage_mask + ((size_t)b * p.stage_tiles + st.stage_index(t)) * 4);
                }
                if (!warp_wait(sm, &sm.info_empty[u % INFO], ((u / INFO) + 1) & 1, p.status)) break;
                if (lane == 0) {
                    sm.info_mask[u % INFO] = mask;
                    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(&sm.info_full[u % INFO])) : "memory");
                }
            }
            __syncwarp();
        }
    } else if ((warp == 1 || warp == 2) && rank == 0 && n_tiles > 0) {
        // ------------------------------------------------ MMA issuers (even CTA)
        // Warp 1 issues S = Q K^T, warp 2 issues O += P V.  Each commits only its
        // own MMAs, so neither chain waits behind the other's operands.
        // Descriptors are built once; a byte offset o within shared memory is
        // o >> 4 added to the descriptor's start-address field.
        constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, NTILE, false, false);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);
        constexpr uint64_t K16 = 32 >> 4;
        bool ok = true;
        if (warp == 1) {
            constexpr uint64_t Q_CHUNK = (HPC * 128) >> 4, K_CHUNK = (32 * 128) >> 4, K_STAGE = K_BYTES >> 4;
            const uint64_t qd0 = smem_desc_sw128(smem_addr(sm.q[0]), 16, 1024);
            const uint64_t kd0 = smem_desc_sw128(smem_addr(sm.k[0][0]), 16, 1024);
            if (p.stall) ok = warp_wait(sm, &sm.never, 0, p.status, TEST_STALL_NS);
            ok = ok && warp_wait(sm, &sm.q_full, 0, p.status);
            if (ok && lane == 0) sm.q_seen = 1;
            for (int u = 0; u < n_tiles && ok; ++u) {      // S(u) = Q K^T
                const int sb = u & 1;
                ok = warp_wait(sm, &sm.s_empty[sb], ((u >> 1) + 1) & 1, p.status) &&
                     warp_wait_cluster(sm, &sm.k_full[sb], (u >> 1) & 1, p.status);
                if (!ok) break;
                if (lane == 0) sm.k_consumed = u + 1;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t d = tmem + TM_S + 32 * sb;
                    const uint64_t kb = kd0 + K_STAGE * sb;
#pragma unroll
                    for (int c = 0; c < KCH; ++c)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_pair_ss(d, qd0 + Q_CHUNK * c + K16 * kk, kb + K_CHUNK * c + K16 * kk, IDESC_QK,
                                         (c | kk) != 0);
                    umma_commit_pair(&sm.k_empty[sb], 0x3);
                    umma_commit_pair(&sm.s_full[sb], 0x3);
                }
                __syncwarp();
            }
        } else {
            constexpr uint64_t P_BUF = (HPC * 128) >> 4, V_STAGE = V_BYTES >> 4, V_J = (2 * NTILE * 128) >> 4;
            constexpr uint64_t V16 = (16 * 128) >> 4;
            const uint64_t pd0 = smem_desc_sw128(smem_addr(sm.p[0]), 16, 1024);
            const uint64_t vd0 = smem_desc_sw128(smem_addr(sm.v[0][0][0]), NTILE * 128, 1024);
            for (int u = 0; u < n_tiles && ok; ++u) {      // O += P V for tile u
                const int sb = u & 1;
                ok = warp_wait(sm, &sm.p_full[sb], (u >> 1) & 1, p.status) &&
                     warp_wait_cluster(sm, &sm.v_full[sb], (u >> 1) & 1, p.status);
                if (!ok) break;
                if (lane == 0) sm.v_consumed = u + 1;
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t vb = vd0 + V_STAGE * sb;
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t b = vb + V_J * j + V16 * kk;
                            umma_pair_ss(tmem + TM_O + 128 * j, pd0 + K16 * kk, b, IDESC_PV, u > 0 || kk > 0);
                            umma_pair_ss(tmem + TM_O + 128 * j, pd0 + P_BUF + K16 * kk, b, IDESC_PV, true);
                        }
                    umma_commit_pair(&sm.v_empty[sb], 0x3);
                    umma_commit_pair(&sm.pv_done[sb], 0x3);
                }
                __syncwarp();
            }
        }
        if (lane == 0) umma_commit_pair(&sm.mma_done, 0x3);
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ softmax + epilogue
        const int L = threadIdx.x - 128;        // TMEM lane of this thread
        const int h = L & 63, half = L >> 6;     // head within the CTA, kv half of the tile
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int u = 0; u < n_tiles; ++u) {
            const int s = u & 1;
            ok = ok && sm.abort_flag == 0;
            if (ok) ok = mbar_wait(&sm.info_full[u % INFO], (u / INFO) & 1, WAIT_NS, &sm.abort_flag);
            const uint32_t vmask = ok ? (uint32_t)(sm.info_mask[u % INFO] >> (32 * half)) : 0u;
            if (ok) ok = mbar_wait(&sm.s_full[s], (u >> 1) & 1, WAIT_NS, &sm.abort_flag);
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
            const bool move = m_new > -INFINITY && (m_ref == -INFINITY || m_new > m_ref + RESCALE_LOG2);
            const float alpha = !move ? 1.f : (m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_new));
            if (move) {
                l *= alpha;
                m_ref = m_new;
            }
            // P = hi + lo, both bf16: rounding P to one bf16 alone leaves a relative error
            // of 2^-9 on every weight, which peaked rows carry straight into the output.
            float psum = 0.f;
            uint32_t pk_hi[16], pk_lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = exp2f(sv[2 * i] - m_ref), p1 = exp2f(sv[2 * i + 1] - m_ref);
                const float q0 = m_ref == -INFINITY ? 0.f : p0, q1 = m_ref == -INFINITY ? 0.f : p1;
                psum += q0 + q1;
                const __nv_bfloat162 hi = __floats2bfloat162_rn(q0, q1);
                pk_hi[i] = *reinterpret_cast<const uint32_t *>(&hi);
                pk_lo[i] = pack_bf16x2(q0 - __low2float(hi), q1 - __high2float(hi));
            }
            l += psum;
            // The P buffers are rewritten and O may be rescaled: P.V of tile u-1 must be done.
            if (u > 0 && ok) {
                ok = mbar_wait(&sm.pv_done[(u - 1) & 1], ((u - 1) >> 1) & 1, WAIT_NS, &sm.abort_flag);
                if (!ok && sm.abort_flag == 0) set_abort(sm, p.status);
            }
            // tcgen05.ld / st are warp-collective: the whole warp takes the rescale when
            // any of its rows moves its reference, the other rows scale by 1.
            if (__any_sync(0xffffffffu, move) && u > 0) {
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
            uint8_t *prow_hi = sm.p[0] + h * 128, *prow_lo = sm.p[1] + h * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int chunk = 4 * half + c, off = (chunk ^ (h & 7)) << 4;
                *reinterpret_cast<uint4 *>(prow_hi + off) =
                    make_uint4(pk_hi[4 * c], pk_hi[4 * c + 1], pk_hi[4 * c + 2], pk_hi[4 * c + 3]);
                *reinterpret_cast<uint4 *>(prow_lo + off) =
                    make_uint4(pk_lo[4 * c], pk_lo[4 * c + 1], pk_lo[4 * c + 2], pk_lo[4 * c + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_barrier(1, 128);
            if (L == 0) mbar_arrive_cluster(map_to_rank(&sm.p_full[s], 0));
        }
        // ---- epilogue: wait for the last P.V, then write the partial
        if (n_tiles > 0 && ok) {
            ok = mbar_wait(&sm.pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, WAIT_NS, &sm.abort_flag);
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
        // O leaves tensor memory 32 columns at a time (one head row per thread); each warp passes
        // its 32 x 32 block through shared memory (the P buffers, free once the last P.V is
        // done; 16-byte pieces XOR-swizzled by row), so that every store instruction writes
        // four whole 128-byte row pieces instead of 32 scattered 16-byte pieces.
        float *xbuf = reinterpret_cast<float *>(sm.p[0]) + (warp & 3) * 1024;
        const size_t prow0 = ((size_t)b * p.n_splits + split) * HQ + HPC * (int)rank + (32 * (warp & 3) & 63);
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
#pragma unroll
            for (int i = 0; i < 8; ++i)
                *reinterpret_cast<uint4 *>(xbuf + lane * 32 + 4 * ((i ^ lane) & 7)) =
                    make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            __syncwarp();
            // O columns 0..127 hold values 0..255 split by lane half; 128..255 hold 256..511
            const int col = 256 * (q >> 2) + 128 * half + (q & 3) * 32 + 4 * (lane & 7);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int r = 4 * k + (lane >> 3);
                const float4 v = *reinterpret_cast<const float4 *>(xbuf + r * 32 + 4 * (((lane & 7) ^ r) & 7));
                *reinterpret_cast<float4 *>(p.o_part + (prow0 + r) * DV + col) = v;
            }
            __syncwarp();
        }
        tc_fence_before();
    }

    // ---- teardown: every MMA finished before TMEM is released; no CTA leaves early
    if (warp == 3 && n_tiles > 0) {
        // each of the even CTA's two MMA threads commits mma_done to both CTAs after its last MMA
        if (lane == 0 && !mbar_wait(&sm.mma_done, 0, WAIT_NS)) set_abort(sm, p.status);
        __syncwarp();
    }
    __syncthreads();
    cluster_sync();   // neither CTA issues another copy from here on
    // set_abort writes the flag into both CTAs before this barrier, so both read the same
    // value here from their own shared memory (no read of the peer: it may leave after the
    // barrier unless both take the abort path, which ends with a second barrier).
    if (sm.abort_flag) {
      if (rank == 0 && threadIdx.x == 0 && n_tiles > 0) {
        // After an abort, every TMA load either CTA issued lands before either CTA leaves:
        // Q (issued by both producers before their loops), and per stage the last K and V
        // tiles whose full phase no issuer saw complete.  Where only one CTA issued that
        // tile, this thread arrives in place of the other, so the phase completes once the
        // issued bytes have landed.  Every wait is bounded.
        if (!sm.q_seen) (void)mbar_wait(&sm.q_full, 0, WAIT_NS);
        for (int s = 0; s < STAGES; ++s) {
            drain_stage(&sm.k_full[s], sm.last_k_tma[s], ld_peer_s32(&sm.last_k_tma[s]), sm.k_consumed);
            drain_stage(&sm.v_full[s], sm.last_v_tma[s], ld_peer_s32(&sm.last_v_tma[s]), sm.v_consumed);
        }
      }
      cluster_sync();   // the odd CTA leaves only after the drain
    }
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

// bf16 tensor map of `rank` dimensions (dims[0] innermost, strides in bytes for
// dims 1..rank-1), 128-byte swizzle, zero fill outside the tensor.
static bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const uint64_t *strides,
                     const uint32_t *box) {
    EncodeTiled enc = encoder();
    if (!enc) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) { d[i] = dims[i]; bx[i] = box[i]; es[i] = 1; }
    for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Splits per sequence: one CTA pair each, all co-resident; a single sequence takes half the
// pairs (37 splits measured 3 % faster than 74 on the 512K workload: half the partials to merge).
int max_splits(int B) {
    const int clusters = sm_count() / 2;
    return max(1, min(clusters / max(B, 1), clusters / 2));
}

// Staging slots per sequence that a call may need: every top-k tile plus every
// window tile (a window that does not start on a chunk boundary is staged whole).
int stage_tiles(int k, int max_window_len) { return (k + NTILE - 1) / NTILE + (max_window_len + NTILE - 1) / NTILE + 1; }
size_t stage_bytes(int B, int k, int max_window_len) {
    // staged rows, then one 64-bit validity mask per staged tile
    return (size_t)B * stage_tiles(k, max_window_len) * (NTILE * DQK * 2 + 8);
}

int launch(const uint16_t *q, const uint16_t *kv_pool, int64_t k_stride, int64_t n_slots, const int32_t *table,
           int table_stride, const int32_t *topk_idx, const int32_t *topk_count, int k, const int32_t *window_start,
           const int32_t *window_len, int max_window_len, int B, float scale, int n_splits, float *o_part,
           float *m_part, float *l_part, uint8_t *stage, int32_t *status, cudaStream_t stream) {
    // Column chunk c of a row is 128 bytes at offset 128 c, so a row is also a
    // [9][64] array and boxes can span chunks as a third (and fourth) dimension:
    //   K: {64 columns, rows, 9 chunks}, box {64, 32, 9}  -> [chunk][32 rows][128 B]
    //   V: {64 columns, rows, 4 chunks, 2 groups of 4}, box {64, 64, 2, 2} at chunk 2r
    //      -> [group j][chunk 4j + 2r + a][64 rows][128 B]
    //   Q: {64 columns, B x 128 heads, 9 chunks}, box {64, 64, 9}
    CUtensorMap k_map, v_map, ks_map, vs_map, q_map;
    const uint64_t pool_rows = (uint64_t)n_slots * LSA_CHUNK;
    const int G = stage_tiles(k, max_window_len);
    const uint64_t stage_rows = (uint64_t)B * G * NTILE;
    if (pool_rows + 64 >= (1ull << 31) || (uint64_t)B * HQ >= (1ull << 31) || stage_rows >= (1ull << 31))
        return fail(LSA_ERR_SHAPE, "lsa_sparse_decode: pool rows must stay below 2^31 for the latent kernel");
    const uint64_t rb = (uint64_t)k_stride * 2;
    const uint64_t kd[3] = {64, pool_rows, KCH}, ks[2] = {rb, 128};
    const uint32_t kbox[3] = {64, 32, KCH};
    const uint64_t vd[4] = {64, pool_rows, 4, 2}, vs[3] = {rb, 128, 512};
    const uint32_t vbox[4] = {64, NTILE, 2, 2};
    const uint64_t qd[3] = {64, (uint64_t)B * HQ, KCH}, qs[2] = {DQK * 2, 128};
    const uint32_t qbox[3] = {64, HPC, KCH};
    if (!make_map(&k_map, kv_pool, 3, kd, ks, kbox) || !make_map(&v_map, kv_pool, 4, vd, vs, vbox))
        return fail(LSA_ERR_CUDA, "lsa_sparse_decode: cuTensorMapEncodeTiled failed for the KV pool");
    // the staging buffer: the same boxes over dense rows of DQK elements
    const uint64_t skd[3] = {64, stage_rows, KCH}, sks[2] = {DQK * 2, 128};
    const uint64_t svd[4] = {64, stage_rows, 4, 2}, svs[3] = {DQK * 2, 128, 512};
    if (!make_map(&ks_map, stage, 3, skd, sks, kbox) || !make_map(&vs_map, stage, 4, svd, svs, vbox))
        return fail(LSA_ERR_CUDA, "lsa_sparse_decode: cuTensorMapEncodeTiled failed for the staging buffer");
    if (!make_map(&q_map, q, 3, qd, qs, qbox))
        return fail(LSA_ERR_CUDA, "lsa_sparse_decode: cuTensorMapEncodeTiled failed for q");
    Params prm;
    prm.table = table; prm.topk_idx = topk_idx; prm.topk_count = topk_count;
    prm.window_start = window_start; prm.window_len = window_len;
    prm.pool = reinterpret_cast<const uint8_t *>(kv_pool); prm.row_bytes = (int64_t)rb;
    prm.o_part = o_part; prm.m_part = m_part; prm.l_part = l_part; prm.status = status;
    prm.n_rows_pool = n_slots * LSA_CHUNK; prm.table_stride = table_stride; prm.k = k; prm.n_splits = n_splits;
    prm.stage_tiles = G;
    prm.stage_mask = reinterpret_cast<uint16_t *>(stage + (size_t)B * G * NTILE * DQK * 2);
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.stall = take_test_stall(LSA_TEST_STALL_ATTENTION);
    stage_kernel<<<dim3(4 * G, B), STAGE_THREADS, 0, stream>>>(prm, stage);
    int rc = check_launch("stage_kernel");
    if (rc) return rc;
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
    LSA_CUDA(cudaLaunchKernelEx(&cfg, mla_decode_kernel, k_map, v_map, ks_map, vs_map, q_map, prm));
    return LSA_OK;
}

}  // namespace mla2
}  // namespace lsa
