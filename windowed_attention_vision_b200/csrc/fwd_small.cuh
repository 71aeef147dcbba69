// Persistent, warp-specialised forward for windows of at most 128 tokens
// (every query tile has exactly one key tile): the HBM-bound regime of small
// windows (M = 8 in Swin's stage 1 at patch 4, "FLASHSWIN" page, section
// "무엇과 다른가": the fused kernel's overhead is not amortised there, so the
// kernel has to run at memory speed).
//
// One CTA per SM walks a static stride of work items; an item is one 128-row
// tile (a pack of floor(128/N) windows of one head, or one window) and items
// are ordered pack-major, head-minor so that the heads of a token - which
// share its DRAM lines - are read by neighbouring CTAs at the same time.
//
// Roles (4 compute warpgroups + 1 loader warp at d = 32; 3 + 1 at d = 64):
//   loader warp  TMA mode (windows that split into whole swizzle atoms):
//                tensor-map box loads of each window's Q, K, V head slices
//                straight into the swizzled operand tiles - one box for an
//                interior window, two on the wrap seam's row or column, four
//                for the corner window - issued by several lanes at once.
//                Otherwise: cp.async gathers of 16-byte chunks (rank-r
//                factors too).
//   compute warpgroups, item k going to group k % groups: each thread owns
//                one tile row (TMEM lane): it resolves its row's token
//                (window-local coordinates, original position, wrap label),
//                applies window-local RoPE to its Q and K rows in place (fp32,
//                Q scaled by d^-1/2); after a group barrier one elected thread
//                issues S = Q~ K~^T into the group's TMEM columns; every
//                thread then runs max / exp / sum over its window's keys and
//                writes P (bf16 pairs) over the consumed S columns; after a
//                second barrier the elected thread issues O = P V (P read from
//                TMEM); once O lands each thread normalises its row and
//                stores it to the token's original (un-shifted) position.
// TMEM: 128 columns per group - S (fp32, 128 cols), then P over S[0, 64) and
// O over S[64, 64 + d).
// Every wait is bounded; a timeout sets a CTA-wide abort flag and the device
// status word; a group leaves its loop only at a group barrier, all together.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "geometry.cuh"
#include "ptx.cuh"
#include "waits.cuh"

namespace winattn {

// Compute warpgroups per CTA: four for d = 32; three for d = 64, whose rows
// need more registers (the CTA's register file is shared by all roles).
template <int D>
struct SmallRoles {
    static constexpr int kGroups = D <= 32 ? 4 : 3;
    static constexpr int kThreads = (kGroups * 4 + 1) * 32;
    static constexpr int kLoaderWarp = kGroups * 4;
};

// Largest RoPE (cos, sin) table the small-window kernel keeps in shared
// memory: heads * M * (d/4) * 8 bytes.
constexpr uint32_t kSmallTableMax = 8 * 1024;

template <int D, int R>
struct SmallLayout {
    static constexpr uint32_t QC = 0;                       // query content  [128][D] bf16, swizzled
    static constexpr uint32_t QB = QC + 256 * D;            // query factors  [128][R]
    static constexpr uint32_t KC = QB + 256 * R;            // key content    [128][D]
    static constexpr uint32_t KB = KC + 256 * D;            // key factors    [128][R]
    static constexpr uint32_t VO = KB + 256 * R;            // values         [128][D]
    static constexpr uint32_t CODES = VO + 256 * D;         // mask code per tile row, u16[128]
    static constexpr uint32_t OFFS = CODES + 256;           // loader's row offsets (cp.async mode), i64[128]
    static constexpr uint32_t STAGE = (OFFS + 128 * 8 + 1023) & ~1023u;
    // ring depth: as many stages as fit beside a RoPE table of up to
    // kSmallTableMax bytes, at most 8
    static constexpr int NS_FIT = (int)((216u * 1024 - kSmallTableMax) / STAGE);
    // a whole number of rounds of the compute groups, so that tiles k and
    // k + NS (which share a stage) fall to the same group: mbarrier waits
    // test a phase's parity only, and a group must not reach a stage's next
    // phase while an earlier phase is still pending for another group
    static constexpr int NS_CAP = NS_FIT < 8 ? NS_FIT : 8;
    static constexpr int NS = NS_CAP - NS_CAP % SmallRoles<D>::kGroups;
    static constexpr int PF = NS - 2 > 2 ? NS - 2 : 2;      // cp.async mode: items issued ahead
    static constexpr uint32_t IJTAB = NS * STAGE;           // TMA row order: (i << 8 | j) u16[4 kinds][64]
    static constexpr uint32_t TABLE = IJTAB + 512;          // RoPE (cos, sin) [heads][M][D/4]
    static constexpr int kBars = 2 * NS + 3 * SmallRoles<D>::kGroups;
    static __host__ __device__ uint32_t table_bytes(int heads, int M)
    {
        return (uint32_t)(heads * M * (D / 4) * 8 + 15) & ~15u;
    }
    static __host__ __device__ uint32_t bars(int heads, int M) { return TABLE + table_bytes(heads, M); }
    static __host__ __device__ uint32_t bytes(int heads, int M) { return bars(heads, M) + kBars * 8 + 16 + 1024; }
};

// Tensor maps of one operand for the TMA mode: box shapes (width x height in
// tokens) M x M, M/2 x M, M x M/2 and M/2 x M/2.
struct WindowMaps {
    CUtensorMap full, xhalf, yhalf, quarter;
};

// Rows `row` of the swizzled Q and K tiles: both rotated by R(i, j) (when
// table != null; one table read serves both), Q multiplied by `qmul` (when
// scale_q), written back in place, one 16-byte chunk (4 pairs) at a time,
// with packed two-lane fp32 arithmetic.  table4[pos][k/2] holds
// (cos k, cos k+1, sin k, sin k+1) of pos * theta for even k.
template <int D>
__device__ __forceinline__ void rotate_qk_rows(uint8_t *qtile, uint8_t *ktile, int row, const float4 *table4, int i,
                                               int j, bool scale_q, float qmul)
{
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint32_t off = swz_offset(row, c, 2 * D);
        const uint4 uq = *reinterpret_cast<const uint4 *>(qtile + off);
        // pairs (a_e, b_e), e = 0..3, regrouped as (a0, a1), (b0, b1), (a2, a3), (b2, b3)
        float2 qa01 = make_float2(bf16lo(uq.x), bf16lo(uq.y)), qb01 = make_float2(bf16hi(uq.x), bf16hi(uq.y));
        float2 qa23 = make_float2(bf16lo(uq.z), bf16lo(uq.w)), qb23 = make_float2(bf16hi(uq.z), bf16hi(uq.w));
        if (table4) {
            const uint4 uk = *reinterpret_cast<const uint4 *>(ktile + off);
            float2 ka01 = make_float2(bf16lo(uk.x), bf16lo(uk.y)), kb01 = make_float2(bf16hi(uk.x), bf16hi(uk.y));
            float2 ka23 = make_float2(bf16lo(uk.z), bf16lo(uk.w)), kb23 = make_float2(bf16hi(uk.z), bf16hi(uk.w));
            // chunk c holds pairs 4c .. 4c+3 of the head dim: the first half
            // (row coordinate i) or the second half (column coordinate j)
            const bool second = 8 * c >= D / 2;
            const float4 *tp = table4 + (second ? j : i) * (D / 8) + (second ? 2 * c - D / 8 : 2 * c);
            const float4 r01 = tp[0], r23 = tp[1];
            const float2 c01 = make_float2(r01.x, r01.y), s01 = make_float2(r01.z, r01.w);
            const float2 c23 = make_float2(r23.x, r23.y), s23 = make_float2(r23.z, r23.w);
            const float2 n01 = make_float2(-r01.z, -r01.w), n23 = make_float2(-r23.z, -r23.w);
            // (a, b) -> (a cos - b sin, a sin + b cos)
            float2 t;
            t = __ffma2_rn(qb01, n01, __fmul2_rn(qa01, c01));
            qb01 = __ffma2_rn(qb01, c01, __fmul2_rn(qa01, s01));
            qa01 = t;
            t = __ffma2_rn(qb23, n23, __fmul2_rn(qa23, c23));
            qb23 = __ffma2_rn(qb23, c23, __fmul2_rn(qa23, s23));
            qa23 = t;
            t = __ffma2_rn(kb01, n01, __fmul2_rn(ka01, c01));
            kb01 = __ffma2_rn(kb01, c01, __fmul2_rn(ka01, s01));
            ka01 = t;
            t = __ffma2_rn(kb23, n23, __fmul2_rn(ka23, c23));
            kb23 = __ffma2_rn(kb23, c23, __fmul2_rn(ka23, s23));
            ka23 = t;
            uint4 ok;
            ok.x = pack_bf16x2(ka01.x, kb01.x);
            ok.y = pack_bf16x2(ka01.y, kb01.y);
            ok.z = pack_bf16x2(ka23.x, kb23.x);
            ok.w = pack_bf16x2(ka23.y, kb23.y);
            *reinterpret_cast<uint4 *>(ktile + off) = ok;
        }
        if (scale_q) {
            const float2 m2 = make_float2(qmul, qmul);
            qa01 = __fmul2_rn(qa01, m2);
            qb01 = __fmul2_rn(qb01, m2);
            qa23 = __fmul2_rn(qa23, m2);
            qb23 = __fmul2_rn(qb23, m2);
        }
        uint4 oq;
        oq.x = pack_bf16x2(qa01.x, qb01.x);
        oq.y = pack_bf16x2(qa01.y, qb01.y);
        oq.z = pack_bf16x2(qa23.x, qb23.x);
        oq.w = pack_bf16x2(qa23.y, qb23.y);
        *reinterpret_cast<uint4 *>(qtile + off) = oq;
    }
}

// Window kind in the TMA mode: bit 0 = the window straddles the column wrap
// seam (last window column of a shifted map), bit 1 = the row seam.
__device__ __forceinline__ int window_kind(const Geometry &g, int wy, int wx)
{
    if (g.shift == 0)
        return 0;
    return (wx == g.nWx - 1 ? 1 : 0) | (wy == g.nWy - 1 ? 2 : 0);
}

// Window-local (i, j) of row rp of a window of the given kind, in the order
// the TMA boxes land: kind 0 and 2 row-major (two M x M/2 boxes stacked keep
// row-major order); kind 1 two M/2-wide boxes, each row-major; kind 3 four
// M/2 x M/2 quadrants, each row-major.
__device__ __forceinline__ void tma_row_coords(const Geometry &g, int kind, int rp, int &i, int &j)
{
    const int M = g.M, hm = M >> 1;
    if (kind == 1) {
        const int half = M * hm;
        const int bx = rp >= half ? 1 : 0;
        const int r = rp - bx * half;
        i = r / hm;
        j = bx * hm + (r - i * hm);
    } else if (kind == 3) {
        const int q2 = hm * hm;
        const int qd = rp / q2, r = rp - qd * q2;
        const int iy = r / hm;
        i = (qd >> 1) * hm + iy;
        j = (qd & 1) * hm + (r - iy * hm);
    } else {
        i = (int)g.div_M.div((uint32_t)rp);
        j = rp - i * M;
    }
}

// TMA loads apply when every box is a whole number of 8-row swizzle atoms:
// unshifted windows with M*M % 8 == 0, or shift M/2 with (M/2)^2 % 8 == 0;
// packed tiles only (at most 64 tokens per window), no rank-r factors.
__host__ __device__ inline bool small_tma_ok(const Geometry &g)
{
    if (g.rank != 0 || g.U < 2)
        return false;
    if (g.shift == 0)
        return (g.N % 8) == 0;
    return 2 * g.shift == g.M && ((g.shift * g.shift) % 8) == 0;
}

// Tensor map of one operand for a window kind (see window_kind).
__device__ __forceinline__ const CUtensorMap *pick_map(const WindowMaps &m, int kind)
{
    switch (kind) {
    case 1: return &m.xhalf;
    case 2: return &m.yhalf;
    case 3: return &m.quarter;
    default: return &m.full;
    }
}

template <int D, int R, bool TMA>
__global__ void __launch_bounds__(SmallRoles<D>::kThreads, 1)
    winattn_fwd_small_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                             const __nv_bfloat16 *__restrict__ v, const float *__restrict__ theta,
                             const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ out,
                             const Geometry g, const float scale, const __grid_constant__ WindowMaps tm_q,
                             const __grid_constant__ WindowMaps tm_k, const __grid_constant__ WindowMaps tm_v)
{
    using L = SmallLayout<D, R>;
    constexpr int NS = L::NS, PF = L::PF, NW = SmallRoles<D>::kGroups;
    constexpr int kLoaderWarp = SmallRoles<D>::kLoaderWarp;
    static_assert(NS >= 3, "ring too shallow");
    static_assert(NS % NW == 0, "a ring stage must always be consumed by the same compute group");
    static_assert(!TMA || R == 0, "TMA loads carry no rank-r factors");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    uint16_t *ijtab = reinterpret_cast<uint16_t *>(base + L::IJTAB);
    float2 *table = reinterpret_cast<float2 *>(base + L::TABLE);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::bars(g.heads, g.M));
    uint64_t *full = bars, *empty = bars + NS;
    uint64_t *s_full = bars + 2 * NS, *o_full = s_full + NW, *fin = o_full + NW;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::kBars);
    volatile uint32_t *abort_flag = tslot + 1;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int n_items = (int)g.items;
    const int first = blockIdx.x, stride = gridDim.x;
    const int count = first < n_items ? (n_items - 1 - first) / stride + 1 : 0;
    const int table_per_head = g.M * (D / 4);

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (t == 32) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], TMA ? 1 : 32);
            mbar_init(&empty[s], 1);
        }
        for (int w = 0; w < NW; ++w) {
            mbar_init(&s_full[w], 1);
            mbar_init(&o_full[w], 1);
            mbar_init(&fin[w], 1);
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (theta) {
        // table4[h][pos][k/2] = (cos k, cos k+1, sin k, sin k+1) of pos * theta_h
        float *tf = reinterpret_cast<float *>(table);
        for (int idx = t; idx < g.heads * table_per_head; idx += blockDim.x) {
            const int h = idx / table_per_head, r = idx - h * table_per_head;
            const int c = r / (D / 4), kk = r - c * (D / 4);
            float sn, cs;
            sincosf((float)c * __ldg(theta + h * (D / 4) + kk), &sn, &cs);
            float *e = tf + 2 * ((h * g.M + c) * (D / 4) + (kk & ~1));
            e[kk & 1] = cs;
            e[2 + (kk & 1)] = sn;
        }
    }
    if (TMA) {
        for (int idx = t; idx < 4 * g.N; idx += blockDim.x) {
            const int kind = idx / g.N, rp = idx - kind * g.N;
            int i, j;
            tma_row_coords(g, kind, rp, i, j);
            ijtab[kind * 64 + rp] = (uint16_t)((i << 8) | j);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    if (warp == kLoaderWarp && TMA) {
        // ------------------------------------------------------------ loader (TMA)
        if (lane == 0) {
            for (int kind = 0; kind < 4; ++kind) {
                tma_prefetch_map(pick_map(tm_q, kind));
                tma_prefetch_map(pick_map(tm_k, kind));
                tma_prefetch_map(pick_map(tm_v, kind));
            }
        }
        const int M = g.M, hm = M >> 1;
        const int my_slot = lane >> 2, my_box = lane & 3;
        for (int kk = 0; kk < count; ++kk) {
            const int s = kk % NS;
            if (kk >= NS && !warp_wait(&empty[s], ((kk / NS) - 1) & 1, abort_flag))
                break;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const uint32_t sst = sbase + s * L::STAGE;
            const int64_t left = g.wph - (int64_t)it.pack * g.U;
            const int nvalid = left < g.U ? (int)left : g.U;
            if (lane == 0)
                mbar_arrive_expect_tx(&full[s], (uint32_t)(3 * nvalid * g.N * 2 * D));
            __syncwarp();
            if (my_slot < nvalid) {
                const int w = it.pack * g.U + my_slot;
                const int b = (int)g.div_img.div((uint32_t)w);
                const int rem = w - b * g.nWy * g.nWx;
                const int wy = (int)g.div_nWx.div((uint32_t)rem);
                const int wx = rem - wy * g.nWx;
                const int kind = window_kind(g, wy, wx);
                const int nbox = kind == 3 ? 4 : (kind ? 2 : 1);
                if (my_box < nbox) {
                    const int bi = my_box;
                    // rolled-local origin of the box, then its original position
                    const int iy0 = (kind & 2) ? ((kind == 3 ? bi >> 1 : bi) * hm) : 0;
                    const int jx0 = (kind & 1) ? ((kind == 3 ? bi & 1 : bi) * hm) : 0;
                    int y0 = wy * M + iy0 + g.shift;
                    if (y0 >= g.H) y0 -= g.H;
                    int x0 = wx * M + jx0 + g.shift;
                    if (x0 >= g.W) x0 -= g.W;
                    const uint32_t roff = (uint32_t)((my_slot * g.N + bi * (g.N / nbox)) * 2 * D);
                    int c0 = it.h * D;
                    int bb = b;
                    debug_box(c0, x0, y0, bb, D, g.heads * D, (kind & 1) ? hm : M, (kind & 2) ? hm : M, g.W, g.H,
                              g.B);
                    tma_load_4d(sst + L::QC + roff, pick_map(tm_q, kind), c0, x0, y0, bb, &full[s]);
                    tma_load_4d(sst + L::KC + roff, pick_map(tm_k, kind), c0, x0, y0, bb, &full[s]);
                    tma_load_4d(sst + L::VO + roff, pick_map(tm_v, kind), c0, x0, y0, bb, &full[s]);
                }
            }
        }
    } else if (warp == kLoaderWarp) {
        // ------------------------------------------------------------ loader (cp.async)
        constexpr int CD = D / 8, CR = R / 8;
        auto issue = [&](int kk) -> bool {
            const int s = kk % NS;
            if (kk >= NS && !warp_wait(&empty[s], ((kk / NS) - 1) & 1, abort_flag))
                return false;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            uint8_t *st = base + s * L::STAGE;
            const uint32_t sst = sbase + s * L::STAGE;
            int64_t *offs = reinterpret_cast<int64_t *>(st + L::OFFS);
#pragma unroll
            for (int r4 = 0; r4 < 4; ++r4) {
                const int row = r4 * 32 + lane;
                const RowRef rr = tile_row(g, it.pack, 0, row);
                offs[row] = rr.valid ? token_ref(g, rr.w, rr.p, it.h).offset : int64_t(-1);
            }
            __syncwarp();
#pragma unroll 4
            for (int idx = lane; idx < 128 * CD; idx += 32) {
                const int row = idx / CD, ch = idx % CD;
                const int64_t ro = offs[row];
                const uint32_t off = swz_offset(row, ch, 2 * D);
                if (ro >= 0) {
                    const int64_t src = ro + ch * 8;
                    cp_async16(sst + L::QC + off, q + src);
                    cp_async16(sst + L::KC + off, k + src);
                    cp_async16(sst + L::VO + off, v + src);
                }
            }
            if constexpr (R > 0) {
                const __nv_bfloat16 *u_h = bias + (int64_t)it.h * 2 * g.N * R;
                const __nv_bfloat16 *w_h = u_h + (int64_t)g.N * R;
#pragma unroll 4
                for (int idx = lane; idx < 128 * CR; idx += 32) {
                    const int row = idx / CR, ch = idx % CR;
                    const RowRef rr = tile_row(g, it.pack, 0, row);
                    const uint32_t off = swz_offset(row, ch, 2 * R);
                    if (rr.valid) {
                        cp_async16(sst + L::QB + off, u_h + rr.p * R + ch * 8);
                        cp_async16(sst + L::KB + off, w_h + rr.p * R + ch * 8);
                    } else {
                        *reinterpret_cast<uint4 *>(st + L::QB + off) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(st + L::KB + off) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            return true;
        };

        // Groups go out one per item, PF - 1 ahead (empty groups past the
        // end keep the count uniform), so waiting until at most PF - 2 are
        // pending covers the oldest item.
        bool failed = false;
        for (int kk = 0; kk < PF - 1; ++kk) {
            if (kk < count && !failed)
                failed = !issue(kk);
            cp_async_commit();
        }
        for (int kc = 0; kc < count && !failed; ++kc) {
            cp_async_wait<PF - 2>();
            fence_proxy_async_smem();
            mbar_arrive(&full[kc % NS]);
            const int kk = kc + PF - 1;
            if (kk < count)
                failed = !issue(kk);
            cp_async_commit();
        }
        cp_async_wait_all();
    } else if (warp < 4 * NW) {
        // ------------------------------------------------------------ compute groups
        const int w = warp >> 2;
        const int row = t - 128 * w;
        const bool elected = row == 0;
        const uint32_t gbase = tmem + w * 128;  // this group's TMEM columns
        const uint32_t region = gbase + ((uint32_t)((warp & 3) * 32) << 16);
        const int r0 = (warp & 3) * 32;
        int c_lo = 0, c_hi = g.N < 128 ? g.N : 128;
        if (g.U > 1) {
            const int s0 = r0 / g.N, s1 = (r0 + 31) / g.N;
            c_lo = s0 * g.N;
            c_hi = (s1 + 1) * g.N < 128 ? (s1 + 1) * g.N : 128;
        }
        const int ch_lo = c_lo >> 5, ch_hi = (c_hi + 31) >> 5;
        const bool aligned = (g.N & 31) == 0;
        // the fast path reads exactly two 32-column chunks: one 64-token window
        const bool two_chunk = aligned && ch_hi - ch_lo == 2;
        // TMA row order with 64-token windows (M = 8): granule-masked softmax
        const bool gran = TMA && g.N == 64;
        constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
        constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
        bool failed = false;
        int issued = 0;  // UMMA batches this thread issued (elected thread only)

        for (int kc = w; kc < count; kc += NW) {
            const int s = kc % NS, j = kc / NW;
            uint8_t *st = base + s * L::STAGE;
            const uint32_t sst = sbase + s * L::STAGE;
            const Item it = decode_item_head_minor(g, first + kc * stride);
            const RowRef rr = tile_row(g, it.pack, 0, row);
            bool wrapped = false;
            int kind = 0;
            TokenRef tk{};
            int code = 0xFFFE;
            float row_sum = 1.f;
            failed = failed || !warp_wait(&full[s], (kc / NS) & 1, abort_flag);
            if (!failed) {
                // ---- resolve this row's token
                if (rr.valid) {
                    int p = rr.p;
                    if (TMA) {
                        const int b = (int)g.div_img.div((uint32_t)rr.w);
                        const int rem = rr.w - b * g.nWy * g.nWx;
                        const int wy = (int)g.div_nWx.div((uint32_t)rem);
                        kind = window_kind(g, wy, rem - wy * g.nWx);
                        const uint32_t ij = ijtab[kind * 64 + rr.p];
                        p = (int)(ij >> 8) * g.M + (int)(ij & 0xFF);
                        wrapped = kind != 0;
                    } else {
                        wrapped = window_wrapped(g, rr.w);
                    }
                    tk = token_ref(g, rr.w, p, it.h);
                    code = (rr.slot << 2) | tk.label;
                }
                reinterpret_cast<uint16_t *>(st + L::CODES)[row] = (uint16_t)code;
                // ---- window-local RoPE on this row's query and key, in place;
                // a row without a token (empty pack slot) is zeroed, so that its
                // value row contributes exact zeros to P V
                if (rr.valid) {
                    if (theta || R > 0)
                        rotate_qk_rows<D>(st + L::QC, st + L::KC, row,
                                          theta ? reinterpret_cast<const float4 *>(table + it.h * table_per_head)
                                                : nullptr,
                                          tk.i, tk.j, R > 0, scale);
                } else {
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        const uint32_t off = swz_offset(row, c, 2 * D);
                        *reinterpret_cast<uint4 *>(st + L::QC + off) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(st + L::KC + off) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(st + L::VO + off) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before_sync();
            // operands and codes of the tile are complete (or someone failed)
            if (named_bar_any(1 + w, 128, failed))
                break;
            if (elected) {
                tc_fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_bf16_ss(gbase, smem_desc(sst + L::QC + ks * 32, 16, 16 * D, swizzle_code(2 * D)),
                                 smem_desc(sst + L::KC + ks * 32, 16, 16 * D, swizzle_code(2 * D)), kIdescS, ks > 0);
#pragma unroll
                for (int ks = 0; ks < R / 16; ++ks)
                    umma_bf16_ss(gbase, smem_desc(sst + L::QB + ks * 32, 16, 16 * R, swizzle_code(2 * R)),
                                 smem_desc(sst + L::KB + ks * 32, 16, 16 * R, swizzle_code(2 * R)), kIdescS, 1);
                umma_commit(&s_full[w]);
                ++issued;
            }
            const uint16_t *codes = reinterpret_cast<const uint16_t *>(st + L::CODES);
            failed = !warp_wait(&s_full[w], j & 1, abort_flag);
            if (!failed) {
                tc_fence_after_sync();
                // scores in log2 units: without rank-r factors Q was not
                // pre-scaled, so d^-1/2 joins log2(e) here
                const float c2 = R > 0 ? kLog2e : scale * kLog2e;
                const int qcode = rr.valid ? code : 0xFFFF;
                // Keys need no per-element test when the row's window fills
                // whole 32-column chunks and is not wrapped.
                const bool fast = !gran && __all_sync(0xffffffffu, two_chunk && rr.valid && !wrapped);
                float l = 0.f;
                if (gran) {
                    // 64-token windows in TMA row order: the boxes of a window
                    // are its wrap-label regions, so the keys a row may see
                    // are whole 16-key granules of its own window (all four
                    // inside, the row's box of two on a seam, its quadrant in
                    // the corner window).  Masked granules get -inf in the
                    // exponent instead of a per-key test.
                    uint32_t gmask = 0u;
                    if (rr.valid)
                        gmask = kind == 0 ? 0xFu : (kind == 3 ? 1u << (rr.p >> 4) : ((rr.p >> 5) ? 0xCu : 0x3u));
                    float x[64];
                    tmem_ld32(region + ch_lo * 32, x);
                    tmem_ld32(region + ch_lo * 32 + 32, x + 32);
                    float gm[4];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float *xg = x + 16 * q4;
                        float a = fmax3(xg[0], xg[1], xg[2]);
#pragma unroll
                        for (int e = 3; e < 15; e += 2)
                            a = fmax3(a, xg[e], xg[e + 1]);
                        gm[q4] = fmaxf(a, xg[15]);
                    }
                    const float ninf = -INFINITY;
                    const float mx = fmaxf(fmax3((gmask & 1u) ? gm[0] : ninf, (gmask & 2u) ? gm[1] : ninf,
                                                 (gmask & 4u) ? gm[2] : ninf),
                                           (gmask & 8u) ? gm[3] : ninf);
                    const float mneg = mx == ninf ? 0.f : -mx * c2;
                    const float2 cc = make_float2(c2, c2);
                    float2 l2 = make_float2(0.f, 0.f);
                    uint32_t pk[32];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float b = ((gmask >> q4) & 1u) ? mneg : ninf;
                        const float2 bb = make_float2(b, b);
#pragma unroll
                        for (int e = 16 * q4; e < 16 * q4 + 16; e += 2) {
                            const float2 z = __ffma2_rn(make_float2(x[e], x[e + 1]), cc, bb);
                            const float2 p = make_float2(fast_exp2(z.x), fast_exp2(z.y));
                            l2 = __fadd2_rn(l2, p);
                            pk[e >> 1] = pack_bf16x2(p.x, p.y);
                        }
                    }
                    l = l2.x + l2.y;
                    uint32_t zero[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        zero[e] = 0u;
                    if (ch_lo == 0) {
                        tmem_st16(region + 0, pk);
                        tmem_st16(region + 16, pk + 16);
                        tmem_st16(region + 32, zero);
                        tmem_st16(region + 48, zero);
                    } else {
                        tmem_st16(region + 0, zero);
                        tmem_st16(region + 16, zero);
                        tmem_st16(region + 32, pk);
                        tmem_st16(region + 48, pk + 16);
                    }
                } else if (fast) {
                    float x[64];
                    tmem_ld32(region + ch_lo * 32, x);
                    tmem_ld32(region + ch_lo * 32 + 32, x + 32);
                    float mx = fmax3(x[0], x[1], x[2]);
#pragma unroll
                    for (int e = 3; e < 63; e += 2)
                        mx = fmax3(mx, x[e], x[e + 1]);
                    mx = fmaxf(mx, x[63]);
                    const float2 cc = make_float2(c2, c2);
                    const float2 mm = make_float2(-mx * c2, -mx * c2);
                    float2 l2 = make_float2(0.f, 0.f);
                    uint32_t pk[32];
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 z = __ffma2_rn(make_float2(x[e], x[e + 1]), cc, mm);
                        const float2 p = make_float2(fast_exp2(z.x), fast_exp2(z.y));
                        l2 = __fadd2_rn(l2, p);
                        pk[e >> 1] = pack_bf16x2(p.x, p.y);
                    }
                    l = l2.x + l2.y;
                    uint32_t zero[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        zero[e] = 0u;
                    if (ch_lo == 0) {
                        tmem_st16(region + 0, pk);
                        tmem_st16(region + 16, pk + 16);
                        tmem_st16(region + 32, zero);
                        tmem_st16(region + 48, zero);
                    } else {
                        tmem_st16(region + 0, zero);
                        tmem_st16(region + 16, zero);
                        tmem_st16(region + 32, pk);
                        tmem_st16(region + 48, pk + 16);
                    }
                } else {
                    float mx = -INFINITY;
                    for (int ch = ch_lo; ch < ch_hi; ++ch) {
                        float x[32];
                        tmem_ld32(region + ch * 32, x);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (codes[ch * 32 + e] == qcode)
                                mx = fmaxf(mx, x[e]);
                    }
                    const float m = (mx == -INFINITY) ? 0.f : mx * c2;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t pk[16];
                        if (ch >= ch_lo && ch < ch_hi) {
                            float x[32];
                            tmem_ld32(region + ch * 32, x);
#pragma unroll
                            for (int e = 0; e < 32; e += 2) {
                                float p0 = fast_exp2(fmaf(x[e], c2, -m));
                                float p1 = fast_exp2(fmaf(x[e + 1], c2, -m));
                                p0 = codes[ch * 32 + e] == qcode ? p0 : 0.f;
                                p1 = codes[ch * 32 + e + 1] == qcode ? p1 : 0.f;
                                l += p0 + p1;
                                pk[e >> 1] = pack_bf16x2(p0, p1);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                pk[e] = 0u;
                        }
                        tmem_st16(region + ch * 16, pk);
                    }
                }
                tmem_wait_st();
                row_sum = l;
            }
            tc_fence_before_sync();
            // every row's P is in TMEM (or someone failed)
            if (named_bar_any(1 + w, 128, failed))
                break;
            if (elected) {
                tc_fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16_ts(gbase + 64, gbase + ks * 8,
                                 smem_desc(sst + L::VO + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D)), kIdescPV,
                                 ks > 0);
                umma_commit(&o_full[w]);
                umma_commit(&empty[s]);
            }
            failed = !warp_wait(&o_full[w], j & 1, abort_flag);
            if (!failed) {
                tc_fence_after_sync();
                float o[D];
#pragma unroll
                for (int c = 0; c < D / 32; ++c)
                    tmem_ld32(region + 64 + c * 32, o + c * 32);
                if (rr.valid) {
                    const float inv = 1.f / row_sum;
                    const float2 i2 = make_float2(inv, inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(out + tk.offset);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        float2 y[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            y[e] = __fmul2_rn(make_float2(o[8 * c + 2 * e], o[8 * c + 2 * e + 1]), i2);
                        uint4 u;
                        u.x = pack_bf16x2(y[0].x, y[0].y);
                        u.y = pack_bf16x2(y[1].x, y[1].y);
                        u.z = pack_bf16x2(y[2].x, y[2].y);
                        u.w = pack_bf16x2(y[3].x, y[3].y);
                        dst[c] = u;
                    }
                }
            }
        }
        // every UMMA this thread issued has completed before TMEM is released
        if (elected && issued) {
            umma_commit(&fin[w]);
            mbar_wait(&fin[w], 0);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace winattn
