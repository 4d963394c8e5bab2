// sparse_decode.cu -- a4: split-K flash-decode attention over the top-k rows
// plus the recent window, merged by log-sum-exp.
// (arXiv 2606.09079: core attention over the selected entries and the most
// recent 8000 tokens, cjcn.com.cn article section 2; gist.science explainer 2.1.)
//
// Grid (n_splits, head groups, B).  A CTA owns HG query heads of one sequence
// and a contiguous range of that sequence's attended rows (top-k rows first,
// then the window).  Tiles of 32 rows are gathered through the chunk table
// with 16-byte cp.async into a multi-stage shared-memory ring (XOR-swizzled
// rows), scores and P.V run on mma.sync (bf16 in, fp32 accumulate), softmax
// is online in the log2 domain.  Each CTA writes an unnormalised partial
// (O, running max, running sum); a merge kernel combines the splits.
#include "common.cuh"
#include "nvtx_range.cuh"

namespace lsa {

template <int HG_, int DQK_, int DV_, int NW_, bool LATENT_>
struct DecodeCfg {
    static constexpr int HG = HG_, DQK = DQK_, DV = DV_, NW = NW_;
    static constexpr bool LATENT = LATENT_;
    static constexpr int NT = NW * 32;
    static constexpr int N = 32;                       // kv rows per tile
    static constexpr int STAGES = LATENT ? 3 : 4;
    static constexpr int WM = HG / 16;                 // 16-head m tiles
    static constexpr int WN = NW / WM;                 // warps sharing one m tile
    static constexpr int NS = N / WN / 8;              // score n8 tiles per warp
    static constexpr int NO = DV / WN / 8;             // output n8 tiles per warp
    static constexpr int KROW = DQK * 2;               // bytes of one K row
    static constexpr int VROW = LATENT ? KROW : DV * 2;
    static constexpr int KCH = KROW / 16, VCH = DV * 2 / 16;   // 16-byte chunks per row
    static constexpr int K_BYTES = N * KROW;
    static constexpr int STAGE_BYTES = K_BYTES + (LATENT ? 0 : N * VROW);
    static constexpr int Q_BYTES = HG * KROW;
    static constexpr int P_BYTES = HG * N * 2;
    static constexpr int TPR = NT / N;                 // loader threads per row
    static constexpr int LOAD_CH = LATENT ? KCH : KCH + VCH;
    static constexpr size_t SMEM = (size_t)Q_BYTES + (size_t)STAGES * STAGE_BYTES + P_BYTES +
                                   sizeof(float) * WN * HG * 2 + sizeof(int) * STAGES * N + 128;
    static_assert(HG % 16 == 0 && NW % WM == 0 && N % (WN * 8) == 0 && (DV / WN) % 16 == 0, "bad tiling");
    static_assert(NS == 1 || NS % 2 == 0, "score tiles");
    static_assert(KROW % 128 == 0 && (LATENT || VROW % 128 == 0), "rows must be 128-byte multiples");
    static_assert(NT % N == 0, "loader mapping");
};

// P tile [HG][32] bf16: 64-byte rows; chunk index XOR (row/2)%4 keeps eight
// consecutive rows on eight different bank groups.
__device__ __forceinline__ uint32_t p_off(int r, int c) { return uint32_t(r * 64 + ((c ^ ((r >> 1) & 3)) << 4)); }

template <class C>
__global__ void __launch_bounds__(C::NT, 1)
sparse_decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k_pool, int64_t k_stride,
                     const uint16_t *__restrict__ v_pool, int64_t v_stride, int64_t n_slots,
                     const int32_t *__restrict__ table, int table_stride, const int32_t *__restrict__ topk_idx,
                     const int32_t *__restrict__ topk_count, int k, const int32_t *__restrict__ window_start,
                     const int32_t *__restrict__ window_len, int Hq, float scale_log2, int n_splits,
                     float *__restrict__ o_part, float *__restrict__ m_part, float *__restrict__ l_part,
                     int32_t *status) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((128 - (smem_addr(smem_raw) & 127)) & 127);
    unsigned char *sQ = base;
    unsigned char *sKV = sQ + C::Q_BYTES;
    unsigned char *sP = sKV + C::STAGES * C::STAGE_BYTES;
    float *red_max = reinterpret_cast<float *>(sP + C::P_BYTES);   // [WN][HG]
    float *red_sum = red_max + C::WN * C::HG;                         // [WN][HG]
    int *row_ok = reinterpret_cast<int *>(red_sum + C::WN * C::HG);  // [STAGES][N]

    const int split = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int mi = warp % C::WM, ni = warp / C::WM;
    const int g = lane >> 2, qd = lane & 3;

    const int tk = min(max(topk_count[b], 0), k);
    const int wstart = window_start[b];
    const int n_rows = tk + max(window_len[b], 0);
    const int tiles_total = (n_rows + C::N - 1) / C::N;
    const int tiles_per = (tiles_total + n_splits - 1) / n_splits;
    const int r0 = split * tiles_per * C::N;
    const int r1 = min(n_rows, r0 + tiles_per * C::N);
    const int n_tiles = r0 < r1 ? (r1 - r0 + C::N - 1) / C::N : 0;
    const int32_t *trow = table + (size_t)b * table_stride;
    const int32_t *tkrow = topk_idx + (size_t)b * k;

    // ---- query heads of this group -> shared memory
    const uint16_t *qg = q + ((size_t)b * Hq + (size_t)grp * C::HG) * C::DQK;
    for (int i = tid; i < C::HG * C::KCH; i += C::NT) {
        int r = i / C::KCH, c = i % C::KCH;
        cp_async16(sQ + swz(r, c, C::KROW), qg + (size_t)r * C::DQK + c * 8);
    }
    cp_async_commit();

    // ---- tile loader: thread -> (row, chunk set)
    auto issue = [&](int t) {
        if (t < n_tiles) {
            const int stage = t % C::STAGES;
            unsigned char *dst = sKV + stage * C::STAGE_BYTES;
            const int row = tid / C::TPR, sub = tid % C::TPR;
            const int j = r0 + t * C::N + row;
            int64_t prow = -1;
            if (j < r1) {
                const int pos = j < tk ? tkrow[j] : wstart + (j - tk);
                const int chunk = pos >> 6;
                const int slot = (pos >= 0 && chunk < table_stride) ? trow[chunk] : -1;
                if (slot >= 0 && slot < n_slots) prow = (int64_t)slot * LSA_CHUNK + (pos & 63);
                else if (sub == 0) flag(status, pos < 0 ? LSA_DEV_INDEX : LSA_DEV_TABLE);
            }
            if (sub == 0) row_ok[stage * C::N + row] = prow >= 0;
            const uint16_t *ksrc = k_pool + (prow >= 0 ? prow : 0) * k_stride;
            const uint16_t *vsrc = C::LATENT ? ksrc : v_pool + (prow >= 0 ? prow : 0) * v_stride;
            const int bytes = prow >= 0 ? 16 : 0;
            for (int c = sub; c < C::LOAD_CH; c += C::TPR) {
                if (c < C::KCH)
                    cp_async16(dst + swz(row, c, C::KROW), ksrc + c * 8, bytes);
                else
                    cp_async16(dst + C::K_BYTES + swz(row, c - C::KCH, C::VROW), vsrc + (c - C::KCH) * 8, bytes);
            }
        }
        cp_async_commit();
    };

#pragma unroll
    for (int s = 0; s < C::STAGES - 1; ++s) issue(s);

    float o[C::NO][4];
#pragma unroll
    for (int i = 0; i < C::NO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run0 = -INFINITY, m_run1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    const uint32_t qbase = smem_addr(sQ), pbase = smem_addr(sP);
    const int hrow = mi * 16;                       // first head row of this warp's m tile
    const int krow0 = ni * (C::N / C::WN);          // first kv row of this warp's score columns
    const int dvch0 = ni * (C::DV / C::WN) / 8;     // first 16-byte dv chunk of this warp's output

    for (int t = 0; t < n_tiles; ++t) {
        issue(t + C::STAGES - 1);
        cp_async_wait<C::STAGES - 1>();
        __syncthreads();
        const int stage = t % C::STAGES;
        const uint32_t kbase = smem_addr(sKV + stage * C::STAGE_BYTES);
        const uint32_t vbase = C::LATENT ? kbase : kbase + C::K_BYTES;

        // ---- S = Q K^T for this warp's 16 heads x N/WN rows
        float sacc[C::NS][4];
#pragma unroll
        for (int i = 0; i < C::NS; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll 4
        for (int kc = 0; kc < C::KCH; kc += 2) {
            uint32_t a[4];
            ldmatrix_x4(a[0], a[1], a[2], a[3], qbase + swz(hrow + (lane & 15), kc + (lane >> 4), C::KROW));
            if constexpr (C::NS == 1) {
                uint32_t b0, b1;
                ldmatrix_x2(b0, b1, kbase + swz(krow0 + (lane & 7), kc + ((lane >> 3) & 1), C::KROW));
                mma_bf16_16816(sacc[0], a, b0, b1);
            } else {
#pragma unroll
                for (int ns = 0; ns < C::NS; ns += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(b0, b1, b2, b3,
                                kbase + swz(krow0 + ns * 8 + (lane & 7) + ((lane >> 4) << 3), kc + ((lane >> 3) & 1),
                                            C::KROW));
                    mma_bf16_16816(sacc[ns], a, b0, b1);
                    mma_bf16_16816(sacc[ns + 1], a, b2, b3);
                }
            }
        }

        // ---- mask, scale, tile row max
        const int *ok = row_ok + stage * C::N;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int ns = 0; ns < C::NS; ++ns) {
            const int c0 = krow0 + ns * 8 + 2 * qd;
            const bool v0 = ok[c0] != 0, v1 = ok[c0 + 1] != 0;
            sacc[ns][0] = v0 ? sacc[ns][0] * scale_log2 : -INFINITY;
            sacc[ns][1] = v1 ? sacc[ns][1] * scale_log2 : -INFINITY;
            sacc[ns][2] = v0 ? sacc[ns][2] * scale_log2 : -INFINITY;
            sacc[ns][3] = v1 ? sacc[ns][3] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(sacc[ns][0], sacc[ns][1]));
            mx1 = fmaxf(mx1, fmaxf(sacc[ns][2], sacc[ns][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        if constexpr (C::WN > 1) {
            if (qd == 0) {
                red_max[ni * C::HG + hrow + g] = mx0;
                red_max[ni * C::HG + hrow + g + 8] = mx1;
            }
            __syncthreads();
#pragma unroll
            for (int w = 0; w < C::WN; ++w) {
                mx0 = fmaxf(mx0, red_max[w * C::HG + hrow + g]);
                mx1 = fmaxf(mx1, red_max[w * C::HG + hrow + g + 8]);
            }
        }
        const float mn0 = fmaxf(m_run0, mx0), mn1 = fmaxf(m_run1, mx1);
        const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m_run0 - mn0);
        const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m_run1 - mn1);
        m_run0 = mn0;
        m_run1 = mn1;

        // ---- P = exp2(S - m), row sums, P -> shared memory (bf16)
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int ns = 0; ns < C::NS; ++ns) {
            float p0 = mn0 == -INFINITY ? 0.f : exp2f(sacc[ns][0] - mn0);
            float p1 = mn0 == -INFINITY ? 0.f : exp2f(sacc[ns][1] - mn0);
            float p2 = mn1 == -INFINITY ? 0.f : exp2f(sacc[ns][2] - mn1);
            float p3 = mn1 == -INFINITY ? 0.f : exp2f(sacc[ns][3] - mn1);
            ps0 += p0 + p1;
            ps1 += p2 + p3;
            const int col = krow0 + ns * 8 + 2 * qd;
            *reinterpret_cast<uint32_t *>(sP + p_off(hrow + g, col >> 3) + (col & 7) * 2) = pack_bf16x2(p0, p1);
            *reinterpret_cast<uint32_t *>(sP + p_off(hrow + g + 8, col >> 3) + (col & 7) * 2) = pack_bf16x2(p2, p3);
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
#pragma unroll
        for (int i = 0; i < C::NO; ++i) {
            o[i][0] *= al0; o[i][1] *= al0;
            o[i][2] *= al1; o[i][3] *= al1;
        }
        __syncthreads();

        // ---- O += P V for this warp's 16 heads x DV/WN columns
#pragma unroll
        for (int kk = 0; kk < C::N / 16; ++kk) {
            uint32_t a[4];
            ldmatrix_x4(a[0], a[1], a[2], a[3], pbase + p_off(hrow + (lane & 15), kk * 2 + (lane >> 4)));
#pragma unroll
            for (int no = 0; no < C::NO; no += 2) {
                uint32_t b0, b1, b2, b3;
                const int vr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int vc = dvch0 + no + (lane >> 4);
                ldmatrix_x4_trans(b0, b1, b2, b3, vbase + swz(vr, vc, C::VROW));
                mma_bf16_16816(o[no], a, b0, b1);
                mma_bf16_16816(o[no + 1], a, b2, b3);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    // ---- partial results
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (qd == 0) {
        red_sum[ni * C::HG + hrow + g] = l0;
        red_sum[ni * C::HG + hrow + g + 8] = l1;
    }
    __syncthreads();
    const size_t part = ((size_t)b * n_splits + split) * Hq + (size_t)grp * C::HG;
    if (ni == 0 && qd == 0) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int w = 0; w < C::WN; ++w) {
            s0 += red_sum[w * C::HG + hrow + g];
            s1 += red_sum[w * C::HG + hrow + g + 8];
        }
        m_part[part + hrow + g] = m_run0;
        m_part[part + hrow + g + 8] = m_run1;
        l_part[part + hrow + g] = s0;
        l_part[part + hrow + g + 8] = s1;
    }
    float *orow0 = o_part + (part + hrow + g) * C::DV + dvch0 * 8 + 2 * qd;
    float *orow1 = orow0 + 8 * C::DV;
#pragma unroll
    for (int no = 0; no < C::NO; ++no) {
        *reinterpret_cast<float2 *>(orow0 + no * 8) = make_float2(o[no][0], o[no][1]);
        *reinterpret_cast<float2 *>(orow1 + no * 8) = make_float2(o[no][2], o[no][3]);
    }
}

// Combines the split-K partials of each head (the log-sum-exp merge).  DV / 8
// threads per head, two float4 columns each (NV = 2), or DV / 4 threads with one
// each (NV = 1), 128 threads per CTA: grid (Hq / heads per CTA, B).  A split that saw no rows wrote m = -inf, l = 0 and
// O = 0, so every partial row is read without branching.  The loads of up to
// MERGE_GROUP splits are issued together before any arithmetic; a longer split
// list is taken group by group, rescaling the running sums to the new maximum.
// A group of 10 keeps the kernel within 128 registers (four CTAs per
// multiprocessor), so the 512 CTAs of an 8-sequence, 128-head merge are one wave.
constexpr int MERGE_GROUP = 10;

template <int DV, int NV>
__global__ void __launch_bounds__(128, 4) lse_merge_kernel(const float *__restrict__ o_part,
                                                        const float *__restrict__ m_part,
                                                        const float *__restrict__ l_part, int n_splits, int Hq,
                                                        float *__restrict__ out, float *__restrict__ lse) {
    // NV float4 columns per thread: TPH threads per head, HPB heads per CTA
    constexpr int TPH = DV / 4 / NV, HPB = 128 / TPH;
    const int t = threadIdx.x % TPH, h = blockIdx.x * HPB + threadIdx.x / TPH, b = blockIdx.y;
    if (h >= Hq) return;
    const size_t row0 = (size_t)b * n_splits * Hq + h;   // partial row of split s: row0 + s * Hq
    float M = -INFINITY, L = 0.f;
    float4 a[NV];
#pragma unroll
    for (int c = 0; c < NV; ++c) a[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_splits; s0 += MERGE_GROUP) {
        float4 v[MERGE_GROUP][NV];
        float ms[MERGE_GROUP], ls[MERGE_GROUP];
#pragma unroll
        for (int j = 0; j < MERGE_GROUP; ++j) {
            if (s0 + j < n_splits) {
                const size_t idx = row0 + (size_t)(s0 + j) * Hq;
                const float4 *src = reinterpret_cast<const float4 *>(o_part + idx * DV);
#pragma unroll
                for (int c = 0; c < NV; ++c) v[j][c] = __ldcs(src + TPH * c + t);
                ms[j] = __ldg(m_part + idx);
                ls[j] = __ldg(l_part + idx);
            } else {
#pragma unroll
                for (int c = 0; c < NV; ++c) v[j][c] = make_float4(0.f, 0.f, 0.f, 0.f);
                ms[j] = -INFINITY;
                ls[j] = 0.f;
            }
        }
        float Mn = M;
#pragma unroll
        for (int j = 0; j < MERGE_GROUP; ++j) Mn = fmaxf(Mn, ms[j]);
        const float r = M == -INFINITY ? 0.f : exp2f(M - Mn);   // the sums so far are 0 while M = -inf
        L *= r;
#pragma unroll
        for (int c = 0; c < NV; ++c) { a[c].x *= r; a[c].y *= r; a[c].z *= r; a[c].w *= r; }
#pragma unroll
        for (int j = 0; j < MERGE_GROUP; ++j) {
            const float w = ms[j] == -INFINITY ? 0.f : exp2f(ms[j] - Mn);
            L += w * ls[j];
#pragma unroll
            for (int c = 0; c < NV; ++c) {
                a[c].x += w * v[j][c].x; a[c].y += w * v[j][c].y; a[c].z += w * v[j][c].z; a[c].w += w * v[j][c].w;
            }
        }
        M = Mn;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    float4 *dst = reinterpret_cast<float4 *>(out + ((size_t)b * Hq + h) * DV);
#pragma unroll
    for (int c = 0; c < NV; ++c) dst[TPH * c + t] = make_float4(a[c].x * inv, a[c].y * inv, a[c].z * inv, a[c].w * inv);
    if (lse && t == 0)
        lse[(size_t)b * Hq + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

// Two float4 columns per thread, or one where the two-column grid would not fill the GPU
// twice over (few sequences), so that more CTAs share the partials' loads.
template <int DV>
static int launch_merge(const float *o_part, const float *m_part, const float *l_part, int n_splits, int Hq, int B,
                        float *out, float *lse, cudaStream_t stream) {
    constexpr int HPB2 = 128 / (DV / 8), HPB1 = 128 / (DV / 4) > 0 ? 128 / (DV / 4) : 1;
    const int ctas2 = (Hq + HPB2 - 1) / HPB2 * B;
    if (DV / 4 <= 128 && ctas2 < 2 * sm_count())
        lse_merge_kernel<DV, 1><<<dim3((Hq + HPB1 - 1) / HPB1, B), 128, 0, stream>>>(o_part, m_part, l_part,
                                                                                    n_splits, Hq, out, lse);
    else
        lse_merge_kernel<DV, 2><<<dim3((Hq + HPB2 - 1) / HPB2, B), 128, 0, stream>>>(o_part, m_part, l_part,
                                                                                    n_splits, Hq, out, lse);
    return check_launch("lse_merge_kernel");
}

// Merge of R attention results of the same queries over disjoint row sets, each
// already normalised (o_r = softmax-weighted mean over its rows, lse_r = log of
// its exp-sum):  lse = log sum_r exp(lse_r),  out = sum_r exp(lse_r - lse) o_r.
// A part without rows (lse_r = -inf) adds nothing; with no rows at all the
// result is out = 0, lse = -inf.  grid B * Hq, one float4 column group per thread.
__global__ void __launch_bounds__(128) part_merge_kernel(const float *__restrict__ o_parts,
                                                         const float *__restrict__ lse_parts, int R, int BH, int dv,
                                                         float *__restrict__ out, float *__restrict__ lse) {
    const int row = blockIdx.x;   // (b, h)
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, lse_parts[(size_t)r * BH + row]);
    float L = 0.f;
    for (int r = 0; r < R; ++r) {
        const float x = lse_parts[(size_t)r * BH + row];
        L += x == -INFINITY ? 0.f : expf(x - M);
    }
    for (int c = threadIdx.x; c < dv / 4; c += blockDim.x) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < R; ++r) {
            const float x = lse_parts[(size_t)r * BH + row];
            if (x == -INFINITY) continue;
            const float w = expf(x - M) / L;
            const float4 v = reinterpret_cast<const float4 *>(o_parts + ((size_t)r * BH + row) * dv)[c];
            a.x += w * v.x; a.y += w * v.y; a.z += w * v.z; a.w += w * v.w;
        }
        reinterpret_cast<float4 *>(out + (size_t)row * dv)[c] = a;
    }
    if (lse && threadIdx.x == 0) lse[row] = L > 0.f ? M + logf(L) : -INFINITY;
}

using CfgSep16 = DecodeCfg<16, 128, 128, 4, false>;
using CfgMla64 = DecodeCfg<64, 576, 512, 8, true>;

namespace mla2 {
int launch(const uint16_t *q, const uint16_t *kv_pool, int64_t k_stride, int64_t n_slots, const int32_t *table,
           int table_stride, const int32_t *topk_idx, const int32_t *topk_count, int k, const int32_t *window_start,
           const int32_t *window_len, int max_window_len, int B, float scale, int n_splits, float *o_part,
           float *m_part, float *l_part, uint8_t *stage, int32_t *status, cudaStream_t stream);
int max_splits(int B);
size_t stage_bytes(int B, int k, int max_window_len);
}  // namespace mla2

// Sep16: 16 heads, separate K/V rows of 128 (mma.sync).  Mla64: 64 latent heads
// (mma.sync).  Mla128: 128 latent heads on tcgen05 with a CTA pair per split.
enum class Variant { None, Sep16, Mla64, Mla128 };

static Variant pick(int Hq, int dqk, int dv, bool latent) {
    if (!latent && Hq == 16 && dqk == 128 && dv == 128) return Variant::Sep16;
    if (latent && Hq == 128 && dqk == 576 && dv == 512) return Variant::Mla128;
    if (latent && Hq == 64 && dqk == 576 && dv == 512) return Variant::Mla64;
    return Variant::None;
}

template <class C>
static int ctas_per_sm() {
    static int cached = -1;
    if (cached < 0) {
        cudaFuncSetAttribute(sparse_decode_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, sparse_decode_kernel<C>, C::NT, C::SMEM) != cudaSuccess ||
            n < 1)
            n = 1;
        cached = n;
    }
    return cached;
}

template <class C>
static int choose_splits(int B, int Hq, int k, int max_window_len) {
    const int groups = Hq / C::HG;
    const int tiles_max = (k + max_window_len + C::N - 1) / C::N;
    const int target = sm_count() * ctas_per_sm<C>();
    int s = target / (B * groups);
    return max(1, min(s, max(1, tiles_max)));
}

static int splits_for(Variant v, int B, int Hq, int k, int max_window_len) {
    if (v == Variant::Mla128) {
        const int tiles_max = (k + 63) / 64 + (max_window_len + 63) / 64;
        return max(1, min(mla2::max_splits(B), tiles_max));
    }
    return v == Variant::Sep16 ? choose_splits<CfgSep16>(B, Hq, k, max_window_len)
                               : choose_splits<CfgMla64>(B, Hq, k, max_window_len);
}

template <class C>
static int launch(const uint16_t *q, const uint16_t *k_pool, int64_t k_stride, const uint16_t *v_pool,
                  int64_t v_stride, int64_t n_slots, const int32_t *table, int table_stride, const int32_t *topk_idx,
                  const int32_t *topk_count, int k, const int32_t *window_start, const int32_t *window_len, int B,
                  int Hq, float scale, int n_splits, float *o_part, float *m_part, float *l_part, int32_t *status,
                  cudaStream_t stream) {
    ctas_per_sm<C>();  // sets the shared-memory attribute
    dim3 grid(n_splits, Hq / C::HG, B);
    sparse_decode_kernel<C><<<grid, C::NT, C::SMEM, stream>>>(
        q, k_pool, k_stride, v_pool, v_stride, n_slots, table, table_stride, topk_idx, topk_count, k, window_start,
        window_len, Hq, scale * 1.4426950408889634f, n_splits, o_part, m_part, l_part, status);
    return check_launch("sparse_decode_kernel");
}

}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_sparse_decode_workspace_size(int B, int Hq, int dqk, int dv, int k, int max_window_len) {
    Variant v = pick(Hq, dqk, dv, dqk != dv);
    if (v == Variant::None || B <= 0 || k < 0 || max_window_len < 0) return 0;
    const int ns = splits_for(v, B, Hq, k, max_window_len);
    Carver c(nullptr);
    c.take<float>((size_t)B * ns * Hq * dv);
    c.take<float>((size_t)B * ns * Hq);
    c.take<float>((size_t)B * ns * Hq);
    if (v == Variant::Mla128) c.take<uint8_t>(mla2::stage_bytes(B, k, max_window_len));   // staged tiles
    return align_up(c.used, 256);
}

extern "C" int lsa_sparse_decode(const lsa_bf16 *q, const lsa_bf16 *k_pool, int64_t k_row_stride,
                                 const lsa_bf16 *v_pool, int64_t v_row_stride, int64_t n_slots,
                                 const int32_t *chunk_table, int table_stride, const int32_t *topk_idx,
                                 const int32_t *topk_count, int k, const int32_t *window_start,
                                 const int32_t *window_len, int max_window_len, int B, int Hq, int dqk, int dv,
                                 float scale, float *out, float *lse, int32_t *dev_status, void *ws, size_t ws_bytes,
                                 lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(B > 0 && n_slots > 0 && table_stride > 0 && k >= 0 && max_window_len >= 1, LSA_ERR_INVALID_ARG,
                "lsa_sparse_decode: bad sizes (B=%d n_slots=%lld table_stride=%d k=%d max_window_len=%d)", B,
                (long long)n_slots, table_stride, k, max_window_len);
    LSA_REQUIRE(q && k_pool && chunk_table && topk_count && window_start && window_len && out && (k == 0 || topk_idx),
                LSA_ERR_INVALID_ARG, "lsa_sparse_decode: null pointer");
    const bool latent = v_pool == nullptr;
    Variant v = pick(Hq, dqk, dv, latent);
    LSA_REQUIRE(v != Variant::None, LSA_ERR_SHAPE,
                "lsa_sparse_decode: unsupported (Hq=%d, dqk=%d, dv=%d, %s); supported: (16,128,128) separate K/V, "
                "(64|128,576,512) latent",
                Hq, dqk, dv, latent ? "latent" : "separate K/V");
    LSA_REQUIRE(k_row_stride >= dqk && k_row_stride % 8 == 0 && (latent || (v_row_stride >= dv && v_row_stride % 8 == 0)),
                LSA_ERR_INVALID_ARG, "lsa_sparse_decode: row strides must cover the row and be multiples of 8");
    LSA_REQUIRE(scale > 0.f, LSA_ERR_INVALID_ARG, "lsa_sparse_decode: scale must be positive");
    const size_t need = lsa_sparse_decode_workspace_size(B, Hq, dqk, dv, k, max_window_len);
    LSA_REQUIRE(ws && ws_bytes >= need, LSA_ERR_WORKSPACE, "lsa_sparse_decode: workspace of %zu bytes, %zu needed",
                ws_bytes, need);
    const int ns = splits_for(v, B, Hq, k, max_window_len);
    Carver c(ws);
    float *o_part = c.take<float>((size_t)B * ns * Hq * dv);
    float *m_part = c.take<float>((size_t)B * ns * Hq);
    float *l_part = c.take<float>((size_t)B * ns * Hq);
    uint8_t *stage = v == Variant::Mla128 ? c.take<uint8_t>(mla2::stage_bytes(B, k, max_window_len)) : nullptr;
    int rc = v == Variant::Mla128
                 ? mla2::launch(q, k_pool, k_row_stride, n_slots, chunk_table, table_stride, topk_idx, topk_count, k,
                                window_start, window_len, max_window_len, B, scale, ns, o_part, m_part, l_part, stage,
                                dev_status, stream)
             : v == Variant::Sep16
                 ? launch<CfgSep16>(q, k_pool, k_row_stride, v_pool, v_row_stride, n_slots, chunk_table, table_stride,
                                    topk_idx, topk_count, k, window_start, window_len, B, Hq, scale, ns, o_part, m_part,
                                    l_part, dev_status, stream)
                 : launch<CfgMla64>(q, k_pool, k_row_stride, v_pool, v_row_stride, n_slots, chunk_table, table_stride,
                                    topk_idx, topk_count, k, window_start, window_len, B, Hq, scale, ns, o_part, m_part,
                                    l_part, dev_status, stream);
    if (rc) return rc;
    return dv == 512 ? launch_merge<512>(o_part, m_part, l_part, ns, Hq, B, out, lse, stream)
                     : launch_merge<128>(o_part, m_part, l_part, ns, Hq, B, out, lse, stream);
}

extern "C" int lsa_merge_attention(const float *o_parts, const float *lse_parts, int R, int B, int Hq, int dv,
                                   float *out, float *lse, lsa_stream_t stream) {
    LSA_ABI_RANGE();
    LSA_REQUIRE(o_parts && lse_parts && out, LSA_ERR_INVALID_ARG, "lsa_merge_attention: null pointer");
    LSA_REQUIRE(R >= 1 && B >= 1 && Hq >= 1 && dv >= 4 && dv % 4 == 0 && (int64_t)B * Hq < (1 << 30),
                LSA_ERR_INVALID_ARG, "lsa_merge_attention: bad sizes (R=%d B=%d Hq=%d dv=%d)", R, B, Hq, dv);
    part_merge_kernel<<<B * Hq, 128, 0, stream>>>(o_parts, lse_parts, R, B * Hq, dv, out, lse);
    return check_launch("part_merge_kernel");
}
