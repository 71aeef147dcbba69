// Persistent, warp-specialised forward for large windows (M in {16, 32, 64,
// 96}: 256 to 9216 tokens): the compute-bound regime ("FLASHSWIN" page,
// section "어떻게 동작하나": an IO-aware fused kernel accumulates the softmax
// online over key tiles, so the N x N score matrix is never stored; the
// windows grow to 96 x 96 on the "Rank-Factorized Implicit Neural Bias"
// page, section 3).
//
// Work item: one window-head (a "unit") and a pair of 128-row query tiles of
// it; items are ordered unit-major, so the pairs of one window run side by
// side on neighbouring SMs and its keys and values are read from L2.
//
// Key/value tiles are whole rows of the window (BN = 128 tokens, or 96 at
// M = 96), loaded by TMA boxes straight into swizzled operand tiles of a
// ring; when the window straddles the column wrap seam (shift M/2) a tile is
// two boxes of M/2 columns, never a rolled copy.  Query tiles are gathered
// with cp.async in the window's row-major order.
//
// Roles (14 warps):
//   warps 0-3 / 4-7  softmax warpgroups A / B, one per query tile: each
//                    thread owns one query row (TMEM lane), runs the online
//                    softmax over the key tiles (running max m and sum l in
//                    fp32, exp2 in log2 units), writes P (bf16 pairs) over the
//                    consumed S columns, rescales its O row in TMEM only when
//                    the max grows by more than 2^8, and at the end
//                    normalises O and stores it to the token's original
//                    (un-shifted) position;
//   warps 8-11       converter: per item, the RoPE table of the head and the
//                    query tiles (cp.async gather, window-local 2D RoPE in
//                    fp32, d^-1/2 folded in when rank-r factors are present);
//                    per key tile, RoPE on the K rows in place;
//   warp 12          TMA loader of K, V (and the key-side factors w);
//   warp 13          MMA issuer: the steps (key tile, query tile A or B) of all
//                    the CTA's items form one sequence; S of a step is issued
//                    NB steps ahead into a rotating TMEM buffer, right behind
//                    the P V that frees it, so a softmax group finds its next
//                    S already computed; O_A += P_A V, O_B += P_B V as soon as
//                    each P is ready.
// TMEM: NB S buffers of BN fp32 columns (NB = 3 at BN = 128, 4 at BN = 96;
// P as bf16 pairs over the first BN/2 columns of its buffer), then O of tile
// A and of tile B (d columns each), twice at d = 32: items alternate between
// the two O buffers, so an item's epilogue can trail the next item's first
// step.
// Wrap masks are structural: a key tile lies on one side of the row seam,
// and its two boxes on the two sides of the column seam, so each query row
// keeps all, none, or one half of a tile.
// Registers: the CTA launches with 128 per thread; each warpgroup then takes
// its share (softmax 184, converter 80, loader and issuers 64), so a softmax
// thread holds its whole row of S between the max pass and the exp pass.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "geometry.cuh"
#include "ptx.cuh"
#include "waits.cuh"

namespace winattn {

constexpr int kLargeThreads = 16 * 32;
// Register split of a CTA launched with 128 registers per thread: the two
// softmax warpgroups hold a whole row of S (BN fp32 values) in registers
// between the max and the exp pass; the converter and the single-thread roles
// need far fewer.  The shares add up to the launch's total, so no .inc waits.
constexpr uint32_t kLargeRegsLaunch = 128, kLargeRegsSoftmax = 184, kLargeRegsConv = 80, kLargeRegsIssue = 64;
static_assert(2 * 128 * kLargeRegsSoftmax + 128 * kLargeRegsConv + 128 * kLargeRegsIssue ==
                  kLargeThreads * kLargeRegsLaunch,
              "register split must add up to the launch's registers");
constexpr uint32_t kLargeSmemBudget = 220 * 1024;

// Keys per tile: 128 (8, 4 or 2 window rows for M = 16, 32, 64), or one
// window row (96 tokens) for M = 96.
__host__ __device__ inline int large_tile_keys(int M) { return M == 96 ? 96 : 128; }

// Windows this kernel serves (the rest go to the generic kernel): M in
// {16, 32, 64, 96}; shift 0 or M/2 (key tiles then never straddle the row
// seam and split into two equal boxes at the column seam); rank-r factors
// only without a shift.
__host__ __device__ inline bool large_ok(const Geometry &g)
{
    if (g.M != 16 && g.M != 32 && g.M != 64 && g.M != 96)
        return false;
    if (g.shift != 0 && 2 * g.shift != g.M)
        return false;
    return g.rank == 0 || g.shift == 0;
}

template <int D, int R, int BN>
struct LargeLayout {
    static constexpr uint32_t QTILE = 256 * (D + R);             // 128 rows: content [128][D], factors [128][R]
    static constexpr uint32_t QBUF = 2 * QTILE;                   // a pair of query tiles
    static constexpr uint32_t KC = 0;                             // key content  [BN][D]   (in a stage)
    static constexpr uint32_t KB = KC + BN * 2 * D;               // key factors  [BN][R]
    static constexpr uint32_t VO = KB + BN * 2 * R;               // values       [BN][D]
    static constexpr uint32_t STAGE = (VO + BN * 2 * D + 1023) & ~1023u;
    static constexpr uint32_t STAGES = 2 * QBUF;                  // ring start
    static constexpr uint32_t TABLE_BYTES = 96 * D * 2;           // RoPE (cos, sin) float4 [M][D/8], M <= 96
    static constexpr uint32_t FIXED = STAGES + TABLE_BYTES + 64 * 8 + 16 + 1024;
    static constexpr int NS_FIT = (int)((kLargeSmemBudget - FIXED) / STAGE);
    static constexpr int NS = NS_FIT < 8 ? NS_FIT : 8;
    static constexpr uint32_t TABLE = STAGES + NS * STAGE;
    static constexpr uint32_t BARS = TABLE + TABLE_BYTES;
    static constexpr uint32_t BYTES = BARS + 64 * 8 + 16 + 1024;
};

// Row `row` of a swizzled bf16 tile with D content columns: rotated by
// R(i, j) with packed two-lane fp32 arithmetic (table4[pos][k/2] holds
// (cos k, cos k+1, sin k, sin k+1) of pos * theta, even k), optionally
// multiplied by `mul`, written back in place.
template <int D>
__device__ __forceinline__ void rotate_row_f2(uint8_t *tile, int row, const float4 *table4, int i, int j,
                                              bool scale, float mul)
{
    // chunks in groups of G, every load of a group issued before its first
    // store (the stores may alias later loads for all the compiler knows)
    constexpr int NCK = D / 8, G = NCK < 4 ? NCK : 4;
#pragma unroll
    for (int c0 = 0; c0 < NCK; c0 += G) {
        uint4 uu[G];
#pragma unroll
        for (int g = 0; g < G; ++g)
            uu[g] = *reinterpret_cast<const uint4 *>(tile + swz_offset(row, c0 + g, 2 * D));
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int c = c0 + g;
            const uint32_t off = swz_offset(row, c, 2 * D);
            const uint4 u = uu[g];
            float2 a01 = make_float2(bf16lo(u.x), bf16lo(u.y)), b01 = make_float2(bf16hi(u.x), bf16hi(u.y));
            float2 a23 = make_float2(bf16lo(u.z), bf16lo(u.w)), b23 = make_float2(bf16hi(u.z), bf16hi(u.w));
            if (table4) {
                const bool second = 8 * c >= D / 2;
                const float4 *tp = table4 + (second ? j : i) * (D / 8) + (second ? 2 * c - D / 8 : 2 * c);
                const float4 r01 = tp[0], r23 = tp[1];
                const float2 c01 = make_float2(r01.x, r01.y), s01 = make_float2(r01.z, r01.w);
                const float2 c23 = make_float2(r23.x, r23.y), s23 = make_float2(r23.z, r23.w);
                const float2 n01 = make_float2(-r01.z, -r01.w), n23 = make_float2(-r23.z, -r23.w);
                float2 t = __ffma2_rn(b01, n01, __fmul2_rn(a01, c01));
                b01 = __ffma2_rn(b01, c01, __fmul2_rn(a01, s01));
                a01 = t;
                t = __ffma2_rn(b23, n23, __fmul2_rn(a23, c23));
                b23 = __ffma2_rn(b23, c23, __fmul2_rn(a23, s23));
                a23 = t;
            }
            if (scale) {
                const float2 m2 = make_float2(mul, mul);
                a01 = __fmul2_rn(a01, m2);
                b01 = __fmul2_rn(b01, m2);
                a23 = __fmul2_rn(a23, m2);
                b23 = __fmul2_rn(b23, m2);
            }
            uint4 o;
            o.x = pack_bf16x2(a01.x, b01.x);
            o.y = pack_bf16x2(a01.y, b01.y);
            o.z = pack_bf16x2(a23.x, b23.x);
            o.w = pack_bf16x2(a23.y, b23.y);
            *reinterpret_cast<uint4 *>(tile + off) = o;
        }
    }
}

// 8 consecutive 32-bit TMEM columns of this thread's lane, written from v[].
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// Tiled 2-D tensor load (no multicast), bytes counted on *bar.
__device__ __forceinline__ void tma_load_2d(uint32_t dst_smem, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// Tensor maps of the large-window kernel: K and V boxes of (d, M, kr) and
// (d, M/2, kr) tokens, and the key-side factors w as (rank, BN) rows.
struct LargeMaps {
    CUtensorMap k_full, k_half, v_full, v_half, w;
};

// Sets bits [start, start + len) of a 128-bit mask.
__device__ __forceinline__ void set_bit_range(uint32_t (&mk)[4], int start, int len)
{
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
        const int lo = max(start - 32 * wd, 0), hi = min(start + len - 32 * wd, 32);
        if (hi > lo)
            mk[wd] |= (hi - lo == 32 ? 0xFFFFFFFFu : ((1u << (hi - lo)) - 1u)) << lo;
    }
}

// Real keys of key tile jt of window (wy, wx) on a padded grid, as a mask
// over the tile's keys in box order (bit c = key c).  The tile's kr window
// rows start at row y0 and never wrap inside the tile, so its real rows are
// a prefix; in each row the real columns are a prefix of the box (two boxes
// at the column seam: the far side starts at column 0).  Pad positions read
// the TMA fill value and must take no weight.
__device__ __forceinline__ void large_key_mask(const Geometry &g, int wy, int wx, int jt, int kr, int BN,
                                               bool xwrap, uint32_t (&mk)[4])
{
    mk[0] = mk[1] = mk[2] = mk[3] = 0u;
    int y0 = wy * g.M + jt * kr + g.shift;
    if (y0 >= g.Hp)
        y0 -= g.Hp;
    const int vr = min(max(g.H - y0, 0), kr);
    const int x0 = wx * g.M + g.shift;
    if (!xwrap) {
        const int pc = min(max(g.W - x0, 0), g.M);
        for (int ri = 0; ri < vr; ++ri)
            set_bit_range(mk, ri * g.M, pc);
    } else {
        const int hm = g.M >> 1;
        const int pl = min(max(g.W - x0, 0), hm), pr = min(g.W, hm);
        for (int ri = 0; ri < vr; ++ri) {
            set_bit_range(mk, ri * hm, pl);
            set_bit_range(mk, BN / 2 + ri * hm, pr);
        }
    }
}

// Epilogue of one query row of item ke: waits for the item's last P V, writes
// O / l (bf16) to `dst` (the token's original position) and hands the O
// buffer (ke % NOB) back to the P V issuer.
template <int D, int NOB>
__device__ __forceinline__ bool large_epilogue_body(__nv_bfloat16 *dst_row, uint32_t obase, int ke, float le, uint64_t *o_last,
                                            uint64_t *t_free, volatile uint32_t *abort_flag)
{
    if (!warp_wait(o_last, ke & 1, abort_flag))
        return false;
    tc_fence_after_sync();
    const uint32_t oe = obase + (ke % NOB) * 2 * D;
    const float inv = 1.f / le;
    const float2 i2 = make_float2(inv, inv);
    uint4 *dst = reinterpret_cast<uint4 *>(dst_row);  // null for a pad row: loads only (warp-collective)
#pragma unroll
    for (int ch = 0; ch < D / 16; ++ch) {
        float o[16];
        tmem_ld16(oe + ch * 16, o);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float2 y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                y[e] = __fmul2_rn(make_float2(o[8 * hh + 2 * e], o[8 * hh + 2 * e + 1]), i2);
            uint4 u;
            u.x = pack_bf16x2(y[0].x, y[0].y);
            u.y = pack_bf16x2(y[1].x, y[1].y);
            u.z = pack_bf16x2(y[2].x, y[2].y);
            u.w = pack_bf16x2(y[3].x, y[3].y);
            if (dst)
                dst[2 * ch + hh] = u;
        }
    }
    tc_fence_before_sync();
    mbar_arrive(t_free);
    return true;
}

// The same kept out of line, for the deferred epilogue inside the step loop,
// where inlined it would cost the softmax registers.
template <int D, int NOB>
__device__ __noinline__ bool large_epilogue_call(__nv_bfloat16 *dst_row, uint32_t obase, int ke, float le,
                                                 uint64_t *o_last, uint64_t *t_free, volatile uint32_t *abort_flag)
{
    return large_epilogue_body<D, NOB>(dst_row, obase, ke, le, o_last, t_free, abort_flag);
}

// PAD: the grid is padded (maps that are not multiples of M); the softmax
// then masks pad keys per tile.  A separate instantiation, so that the
// unpadded kernel's softmax carries none of it.
template <int D, int R, int BN, bool PAD>
__global__ void __launch_bounds__(kLargeThreads, 1)
    winattn_fwd_large_kernel(const __nv_bfloat16 *__restrict__ q, const float *__restrict__ theta,
                             const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ out,
                             float *__restrict__ lse, const Geometry g, const float scale,
                             const __grid_constant__ LargeMaps maps)
{
    using L = LargeLayout<D, R, BN>;
    constexpr int NS = L::NS;
    // S buffers in TMEM (BN fp32 columns each, rotated over both query tiles),
    // then O of tile A and of tile B (D columns each)
    constexpr int NB = BN == 96 ? 4 : 3;
    constexpr uint32_t kOCol = NB * BN;
    // O buffers per query tile: two where TMEM has room (d = 32), so that an
    // item's epilogue can wait behind the next item's first step; one at
    // M = 96, where an item has 96 key tiles and the boundary is rare
    constexpr int NOB = BN == 128 && kOCol + 4 * D <= 512 ? 2 : 1;
    static_assert(kOCol + 2 * NOB * D <= 512, "TMEM columns");
    // S of step n + NB may need key tile cg + NB / 2 while tile cg (step n = 2 cg) is held
    static_assert(NS >= NB / 2 + 1, "ring too shallow for the S lookahead");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    float4 *table4 = reinterpret_cast<float4 *>(base + L::TABLE);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::BARS);
    uint64_t *kv_full = bars, *kv_ready = bars + NS, *kv_empty = bars + 2 * NS;
    // p_part[b * 4 + ch]: chunk ch (32 keys) of the P in S buffer b is written
    uint64_t *q_ready = bars + 3 * NS, *q_free = q_ready + 2, *s_full = q_free + 2, *p_part = s_full + NB;
    uint64_t *pv_done = p_part + 4 * NB, *o_done = pv_done + NB, *o_last = o_done + 2, *t_free = o_last + 2;
    uint64_t *fin = t_free + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(fin + 3);
    volatile uint32_t *abort_flag = tslot + 1;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int M = g.M, N = g.N, kr = BN / M;  // key tile = kr window rows
    const int nkv = N / BN;                   // key tiles per window
    const int npairs = N / 256;               // query-tile pairs per window
    const int n_items = (int)(g.wph * g.heads) * npairs;
    const int first = blockIdx.x, stride = gridDim.x;
    const int count = first < n_items ? (n_items - 1 - first) / stride + 1 : 0;
    const bool has_rope = theta != nullptr;
    // scores in log2 units: without rank-r factors Q is not pre-scaled, so
    // d^-1/2 joins log2(e) in the exponent
    const float c2 = R > 0 ? kLog2e : scale * kLog2e;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (t == 32) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_ready[s], 128);
            mbar_init(&kv_empty[s], 2);  // P V of both query tiles
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&q_ready[a], 128);
            mbar_init(&q_free[a], 1);
            mbar_init(&o_done[a], 1);
            mbar_init(&o_last[a], 1);
            mbar_init(&t_free[a], 128);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&pv_done[b], 1);
            for (int ch = 0; ch < 4; ++ch)
                mbar_init(&p_part[b * 4 + ch], 128);
        }
        for (int f = 0; f < 3; ++f)
            mbar_init(&fin[f], 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    // item -> (window, head, pair); units are head-minor
    auto decode = [&](int kk, int &w, int &h, int &pair) {
        const int item = first + kk * stride;
        const int unit = item / npairs;
        pair = item - unit * npairs;
        w = (int)g.div_heads.div((uint32_t)unit);
        h = unit - w * g.heads;
    };
    auto window_pos = [&](int w, int &b, int &wy, int &wx) {
        b = (int)g.div_img.div((uint32_t)w);
        const int rem = w - b * g.nWy * g.nWx;
        wy = (int)g.div_nWx.div((uint32_t)rem);
        wx = rem - wy * g.nWx;
    };

    // Each warpgroup takes its register share first (one setmaxnreg per
    // warpgroup, at the head of its branch; the host launches this kernel
    // only when it was built with exactly kLargeRegsLaunch registers per
    // thread, so the shares add up).
    if (warp >= 12) {
        warpgroup_regs_dec<kLargeRegsIssue>();
        if (warp == 12) {
            // ============================================================ TMA loader
            if (lane == 0) {
                int c = 0;
                bool ok = true;
                const uint32_t bytes = (uint32_t)(BN * 2 * (2 * D + R));
                for (int kk = 0; kk < count && ok; ++kk) {
                    int w, h, pair, b, wy, wx;
                    decode(kk, w, h, pair);
                    window_pos(w, b, wy, wx);
                    const bool xwrap = g.shift && wx == g.nWx - 1;
                    for (int jt = 0; jt < nkv; ++jt, ++c) {
                        const int s = c % NS;
                        if (c >= NS && !wait_or_abort(&kv_empty[s], ((c / NS) - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t sst = sbase + L::STAGES + s * L::STAGE;
                        mbar_arrive_expect_tx(&kv_full[s], bytes);
                        // rows and columns past H, W (a padded grid) read the
                        // fill value; they are masked in the softmax
                        int y0 = wy * M + jt * kr + g.shift;
                        if (y0 >= g.Hp) y0 -= g.Hp;
                        int x0 = wx * M + g.shift;  // < Wp unless the window straddles the seam
                        int c0 = h * D;
                        // boxes of a padded grid may reach past H, W (fill), never past Hp, Wp
                        debug_box(c0, x0, y0, b, D, g.heads * D, xwrap ? M / 2 : M, kr, g.Wp, g.Hp, g.B);
                        if (xwrap) {
                            const int x1 = 0;             // the seam's far side
                            const uint32_t half = (uint32_t)(BN / 2) * 2 * D;
                            tma_load_4d(sst + L::KC, &maps.k_half, c0, x0, y0, b, &kv_full[s]);
                            tma_load_4d(sst + L::KC + half, &maps.k_half, c0, x1, y0, b, &kv_full[s]);
                            tma_load_4d(sst + L::VO, &maps.v_half, c0, x0, y0, b, &kv_full[s]);
                            tma_load_4d(sst + L::VO + half, &maps.v_half, c0, x1, y0, b, &kv_full[s]);
                        } else {
                            tma_load_4d(sst + L::KC, &maps.k_full, c0, x0, y0, b, &kv_full[s]);
                            tma_load_4d(sst + L::VO, &maps.v_full, c0, x0, y0, b, &kv_full[s]);
                        }
                        if constexpr (R > 0)
                            tma_load_2d(sst + L::KB, &maps.w, 0, (h * 2 + 1) * N + jt * BN, &kv_full[s]);
                    }
                }
                // after an abort no consumer may take the stages armed last:
                // wait (bounded) until their loads have landed, so none is
                // still writing shared memory when the CTA exits
                if (*abort_flag)
                    for (int c2 = c > NS ? c - NS : 0; c2 < c; ++c2)
                        mbar_wait(&kv_full[c2 % NS], (c2 / NS) & 1);
            }
        } else if (warp == 13) {
            // ============================================================ S issuer
            // One sequence over the CTA's items: step n = 2 cg + t is query tile t
            // (0 = A, 1 = B) against the CTA's cg-th key tile.  S of step n goes to
            // TMEM buffer n % NB once P V of step n - NB (the buffer's previous
            // tenant) has completed.
            if (lane == 0) {
                constexpr uint32_t kIdescS = idesc_bf16_f32(128, BN, false);
                const int total = 2 * count * nkv;
                int s_kk = 0, s_jt = 0;  // item and key tile of the next S
                int ns = 0;
                for (; ns < total; ++ns) {
                    const int tl = ns & 1, cg = ns >> 1;
                    if (ns >= NB && !wait_or_abort(&pv_done[ns % NB], ((ns / NB) - 1) & 1, abort_flag))
                        break;
                    if (tl == 0) {
                        if (s_jt == 0 && !wait_or_abort(&q_ready[s_kk & 1], (s_kk >> 1) & 1, abort_flag))
                            break;
                        if (!wait_or_abort(&kv_ready[cg % NS], (cg / NS) & 1, abort_flag))
                            break;
                    }
                    tc_fence_after_sync();
                    const uint32_t qtile = sbase + (s_kk & 1) * L::QBUF + tl * L::QTILE;
                    const uint32_t d = tmem + (ns % NB) * BN;
                    const uint32_t kst = sbase + L::STAGES + (cg % NS) * L::STAGE;
                    // descriptors built once per step; a 16-element K step is
                    // +32 bytes, i.e. +2 in the 16-byte start-address field
                    const uint64_t qd = smem_desc(qtile, 16, 16 * D, swizzle_code(2 * D));
                    const uint64_t kd = smem_desc(kst + L::KC, 16, 16 * D, swizzle_code(2 * D));
    #pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks)
                        umma_bf16_ss(d, qd + 2 * ks, kd + 2 * ks, kIdescS, ks > 0);
                    if constexpr (R > 0) {
                        const uint64_t qbd = smem_desc(qtile + 256 * D, 16, 16 * R, swizzle_code(2 * R));
                        const uint64_t kbd = smem_desc(kst + L::KB, 16, 16 * R, swizzle_code(2 * R));
    #pragma unroll
                        for (int ks = 0; ks < R / 16; ++ks)
                            umma_bf16_ss(d, qbd + 2 * ks, kbd + 2 * ks, kIdescS, 1);
                    }
                    umma_commit(&s_full[ns % NB]);
                    if (tl == 1 && ++s_jt == nkv) {
                        umma_commit(&q_free[s_kk & 1]);  // the last S that reads this item's Q
                        s_jt = 0;
                        ++s_kk;
                    }
                }
                if (ns > 0) {
                    umma_commit(&fin[0]);
                    mbar_wait(&fin[0], 0);
                }
            }
        } else if (warp == 14 || warp == 15) {
            // ============================================================ P V issuers
            // One per query tile: O_t += P V chunk by chunk (32 keys, two MMAs)
            // as the softmax writes each chunk of P, so that P V overlaps the
            // exponentials and the S buffer returns right after the last chunk.
            const int tl = warp - 14;
            if (lane == 0) {
                constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
                constexpr int NC = BN / 32;
                const int steps = count * nkv;
                int p_kk = 0, p_jt = 0;  // item and key tile of this tile's next P V
                int c = 0;
                bool ok = true;
                for (; c < steps && ok; ++c) {
                    const int n = 2 * c + tl, b = n % NB;
                    // O buffer p_kk % NOB of this tile is free once the epilogue of
                    // item p_kk - NOB read it (with two buffers the softmax group
                    // has done that epilogue before it wrote any P of item
                    // p_kk - 1, all of which this issuer has consumed: no phase of
                    // t_free is pending behind the one waited for)
                    if (p_jt == 0 && p_kk >= NOB &&
                        !(ok = wait_or_abort(&t_free[tl], (p_kk - NOB) & 1, abort_flag)))
                        break;
                    // S of this step exists, hence P V of the buffer's previous
                    // tenant (step n - NB, the other tile's) has completed and the
                    // chunk barriers of buffer b are on this step's phase: a
                    // parity wait must never run a phase ahead of its barrier
                    if (!(ok = wait_or_abort(&s_full[b], (n / NB) & 1, abort_flag)))
                        break;
                    const uint32_t pa = tmem + b * BN;  // P over the first BN/2 columns of the buffer
                    const uint32_t vst = sbase + L::STAGES + (c % NS) * L::STAGE + L::VO;
                    const uint32_t od = tmem + kOCol + ((p_kk % NOB) * 2 + tl) * D;
                    // 16 keys of V are 32 D bytes: +2 D in the start-address field
                    const uint64_t vd = smem_desc(vst, 8192, 16 * D, swizzle_code(2 * D));
                    // parts end at chunks 1, 3 (and at the last chunk for BN = 96)
    #pragma unroll
                    for (int ch = 0; ch < NC; ++ch) {
                        if ((ch & 1) || ch == NC - 1) {
                            if (!(ok = wait_or_abort(&p_part[b * 4 + ch], (n / NB) & 1, abort_flag)))
                                break;
                            tc_fence_after_sync();
                            const int c0 = ch & ~1;
    #pragma unroll
                            for (int ks = 2 * c0; ks < 2 * ch + 2; ++ks)
                                umma_bf16_ts(od, pa + ks * 8, vd + (uint64_t)(2 * D * ks), kIdescPV, p_jt > 0 || ks > 0);
                        }
                    }
                    if (!ok)
                        break;
                    umma_commit(&o_done[tl]);
                    if (p_jt == nkv - 1)
                        umma_commit(&o_last[tl]);
                    umma_commit(&pv_done[b]);
                    umma_commit(&kv_empty[c % NS]);
                    if (++p_jt == nkv) {
                        p_jt = 0;
                        ++p_kk;
                    }
                }
                if (c > 0) {
                    umma_commit(&fin[1 + tl]);
                    mbar_wait(&fin[1 + tl], 0);
                }
            }
        }
    } else if (warp >= 8) {
        warpgroup_regs_dec<kLargeRegsConv>();
        // ============================================================ converter
        const int ct = t - 256;
        constexpr int CD = D / 8, CR = R / 8;
        int c = 0;
        bool failed = false;
        // cp.async gather of this thread's two query rows (and factors) of item kk
        auto load_q = [&](int kk) {
            int w, h, pair;
            decode(kk, w, h, pair);
            const uint32_t qbase = sbase + (kk & 1) * L::QBUF;
            for (int t2 = 0; t2 < 2; ++t2) {
                const int p = (2 * pair + t2) * 128 + ct;
                const TokenRef tk = token_ref(g, w, p, h);
                const uint32_t tile = qbase + t2 * L::QTILE;
#pragma unroll
                for (int ch = 0; ch < CD; ++ch)
                    cp_async16(tile + swz_offset(ct, ch, 2 * D), q + tk.offset + ch * 8);
                if constexpr (R > 0) {
                    const __nv_bfloat16 *u = bias + (((int64_t)h * 2 + 0) * N + p) * R;
#pragma unroll
                    for (int ch = 0; ch < CR; ++ch)
                        cp_async16(tile + 256 * D + swz_offset(ct, ch, 2 * R), u + ch * 8);
                }
            }
            cp_async_commit();
        };
        if (count > 0)
            load_q(0);
        for (int kk = 0; kk < count; ++kk) {
            int w, h, pair, b, wy, wx;
            decode(kk, w, h, pair);
            window_pos(w, b, wy, wx);
            const bool xwrap = g.shift && wx == g.nWx - 1;
            const int qb = kk & 1;
            // ---- RoPE table of head h: table4[pos][k/2] = (cos k, cos k+1, sin k, sin k+1)
            if (has_rope) {
                float *tf = reinterpret_cast<float *>(table4);
                for (int idx = ct; idx < M * (D / 4); idx += 128) {
                    const int pos = idx / (D / 4), kq = idx - pos * (D / 4);
                    float sn, cs;
                    sincosf((float)pos * __ldg(theta + h * (D / 4) + kq), &sn, &cs);
                    float *e = tf + 2 * (pos * (D / 4) + (kq & ~1));
                    e[kq & 1] = cs;
                    e[2 + (kq & 1)] = sn;
                }
            }
            cp_async_wait<0>();
            // table built, every query row landed (or someone failed)
            if (named_bar_any(1, 128, failed))
                break;
            // ---- query rows: resolve, rotate (and scale with factors present)
            {
                uint8_t *qbase = base + qb * L::QBUF;
                for (int t2 = 0; t2 < 2; ++t2) {
                    const int p = (2 * pair + t2) * 128 + ct;
                    const TokenRef tk = token_ref(g, w, p, h);
                    if (has_rope || R > 0)
                        rotate_row_f2<D>(qbase + t2 * L::QTILE, ct, has_rope ? table4 : nullptr, tk.i, tk.j, R > 0,
                                         scale);
                }
                fence_proxy_async_smem();
                mbar_arrive(&q_ready[qb]);
            }
            // ---- key tiles: RoPE on K rows in place (TMA row order)
            for (int jt = 0; jt < nkv && !failed; ++jt, ++c) {
                const int s = c % NS;
                if (!warp_wait(&kv_full[s], (c / NS) & 1, abort_flag)) {
                    failed = true;
                    break;
                }
                if (has_rope && ct < BN) {
                    int i, j;
                    if (xwrap) {
                        const int hm = M >> 1, hf = ct >= BN / 2 ? 1 : 0, cc = ct - hf * (BN / 2);
                        const int ri = cc / hm;
                        i = jt * kr + ri;
                        j = hf * hm + (cc - ri * hm);
                    } else {
                        const int ri = ct / M;
                        i = jt * kr + ri;
                        j = ct - ri * M;
                    }
                    rotate_row_f2<D>(base + L::STAGES + s * L::STAGE + L::KC, ct, table4, i, j, false, 1.f);
                }
                fence_proxy_async_smem();
                mbar_arrive(&kv_ready[s]);
            }
            // ---- prefetch the next item's query rows into the other buffer,
            // once the tensor core is done with the item that used it
            if (kk + 1 < count && !failed) {
                if (kk + 1 >= 2 && !warp_wait(&q_free[(kk + 1) & 1], (((kk + 1) >> 1) - 1) & 1, abort_flag))
                    failed = true;
                else
                    load_q(kk + 1);
            }
            // the table may be rebuilt for the next item (or someone failed)
            if (named_bar_any(1, 128, failed))
                break;
        }
        cp_async_wait_all();
    } else {
        warpgroup_regs_inc<kLargeRegsSoftmax>();
        // ============================================================ softmax groups
        const int tile = warp >> 2;  // 0 = A, 1 = B
        const int row = t - 128 * tile;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t obase = tmem + lane_base + kOCol + tile * D;  // O buffer 0 of this tile, this warp's lanes
        constexpr int NCH = BN / 16;                           // 16-column chunks of S
        int c = 0;
        bool failed = false;
        // off < 0: a pad row, nothing is stored
        auto epilogue = [&](int ke, int64_t off, float le) -> bool {
            __nv_bfloat16 *dst = off < 0 ? nullptr : out + off;
            if constexpr (NOB == 2)
                return large_epilogue_call<D, NOB>(dst, obase, ke, le, &o_last[tile], &t_free[tile], abort_flag);
            else
                return large_epilogue_body<D, NOB>(dst, obase, ke, le, &o_last[tile], &t_free[tile], abort_flag);
        };
        // With two O buffers an item's epilogue runs after the first step of
        // the next item, when its last P V has long completed, instead of
        // stalling the group at the item boundary.  Its wait on o_last cannot
        // alias the next item's phase: a window has at least two key tiles,
        // so that phase needs P this group has not yet written.
        int pend_kk = -1;
        int64_t pend_off = 0;
        float pend_l = 1.f;
        for (int kk = 0; kk < count && !failed; ++kk) {
            int w, h, pair, b, wy, wx;
            decode(kk, w, h, pair);
            window_pos(w, b, wy, wx);
            const bool xwrap = g.shift && wx == g.nWx - 1;
            const bool ywrap = g.shift && wy == g.nWy - 1;
            // this thread's query row: token, and its wrap label bits (S of
            // the item implies its query tiles are ready)
            const TokenRef me = token_ref(g, w, (2 * pair + tile) * 128 + row, h);
            const int me_ly = me.label >> 1, me_lx = me.label & 1;
            const uint32_t oreg = obase + (kk % NOB) * 2 * D;  // O of this item
            // Online softmax in log2 units: m is the reference of the row's P
            // (exp2(s * c2 - m)); it moves, rescaling l and O, only when a
            // tile's max exceeds it by more than 2^8.
            float m = -INFINITY, l = 0.f;
            constexpr int NC = BN / 32;  // 32-column chunks of S
            for (int jt = 0; jt < nkv; ++jt, ++c) {
                const int n = 2 * c + tile;  // step of the CTA's S / P sequence
                if (!warp_wait(&s_full[n % NB], (n / NB) & 1, abort_flag)) {
                    failed = true;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t sreg = tmem + lane_base + (n % NB) * BN;  // S (then P) of this step
                // allowed 16-column halves of this row: the tile lies on one
                // side of the row seam, its halves on the two sides of the
                // column seam
                const int ky = ywrap && jt * kr >= (M >> 1) ? 1 : 0;
                int a0 = 0, a1 = NCH;
                if (ky != me_ly) {
                    a0 = a1 = 0;
                } else if (xwrap) {
                    a0 = me_lx ? NCH / 2 : 0;
                    a1 = a0 + NCH / 2;
                }
                // a padded grid: pad keys of this tile (same for every row)
                uint32_t mk[4] = {~0u, ~0u, ~0u, ~0u};
                bool masked = false;
                if constexpr (PAD) {
                    large_key_mask(g, wy, wx, jt, kr, BN, xwrap, mk);
                    masked = (mk[0] & mk[1] & mk[2] & (BN == 128 ? mk[3] : ~0u)) != ~0u;
                }
                // ---- pass 1: the row of S into registers (all loads in
                // flight at once, one wait), then its max over the allowed
                // columns (four independent max chains)
                uint32_t sv[NC][32];
#pragma unroll
                for (int ch = 0; ch < NC; ++ch)
                    tmem_ld32_issue(sreg + ch * 32, sv[ch]);
                tmem_wait_ld32(sv[0]);
#pragma unroll
                for (int ch = 1; ch < NC; ++ch)
                    reg_fence32(sv[ch]);
                if (PAD && masked) {
                    // pad keys: -inf scores, so they weigh nothing
#pragma unroll
                    for (int ch = 0; ch < NC; ++ch)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            sv[ch][e] = ((mk[ch] >> e) & 1u) ? sv[ch][e] : 0xFF800000u;
                }
                float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int ch = 0; ch < NC; ++ch) {
                    const uint32_t *xb = sv[ch];
                    if (2 * ch >= a0 && 2 * ch < a1) {
#pragma unroll
                        for (int e = 0; e < 16; e += 2)
                            mq[(e >> 1) & 3] = fmax3(mq[(e >> 1) & 3], __uint_as_float(xb[e]), __uint_as_float(xb[e + 1]));
                    }
                    if (2 * ch + 1 >= a0 && 2 * ch + 1 < a1) {
#pragma unroll
                        for (int e = 16; e < 32; e += 2)
                            mq[(e >> 1) & 3] = fmax3(mq[(e >> 1) & 3], __uint_as_float(xb[e]), __uint_as_float(xb[e + 1]));
                    }
                }
                const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
                if (PAD && mx == -INFINITY)
                    a0 = a1 = 0;  // nothing of this tile is left after the pad mask
                float alpha = 1.f;
                bool rescale = false;
                if (mx > -INFINITY) {
                    const float mn = mx * c2;
                    if (m == -INFINITY) {
                        m = mn;
                    } else if (mn > m + 8.f) {
                        alpha = fast_exp2(m - mn);
                        m = mn;
                        rescale = true;
                    }
                }
                if (__any_sync(0xffffffffu, rescale)) {
                    // O must hold every earlier key tile's P V before it is
                    // rescaled: only P V of this tile's previous step (c - 1)
                    // can still be in flight.  The rescale lands before the
                    // first chunk of this step's P is handed to P V.
                    if (!warp_wait(&o_done[tile], (c - 1) & 1, abort_flag)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after_sync();
#pragma unroll
                    for (int ch = 0; ch < D / 16; ++ch) {
                        float o[16];
                        tmem_ld16(oreg + ch * 16, o);
                        uint32_t ob[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            ob[e] = __float_as_uint(o[e] * alpha);
                        tmem_st16(oreg + ch * 16, ob);
                    }
                }
                // ---- pass 2: P = exp2(s * c2 - m) from the registers into
                // TMEM over the consumed S; P goes to P V part by part
                const float2 cc = make_float2(c2, c2), mm2 = make_float2(-m, -m);
                float2 lq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // two sum chains
                uint64_t *parts = p_part + (n % NB) * 4;
#pragma unroll
                for (int ch = 0; ch < NC; ++ch) {
                    // P chunk ch covers S columns [16 ch, 16 ch + 16), already read
                    const uint32_t *xb = sv[ch];
                    const bool lo = 2 * ch >= a0 && 2 * ch < a1;
                    const bool hi = 2 * ch + 1 >= a0 && 2 * ch + 1 < a1;
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        if (e < 16 ? lo : hi) {
                            const float2 z = __ffma2_rn(
                                make_float2(__uint_as_float(xb[e]), __uint_as_float(xb[e + 1])), cc, mm2);
                            const float2 p = make_float2(fast_exp2(z.x), fast_exp2(z.y));
                            lq[(e >> 1) & 1] = __fadd2_rn(lq[(e >> 1) & 1], p);
                            pk[e >> 1] = pack_bf16x2(p.x, p.y);
                        } else {
                            pk[e >> 1] = 0u;
                        }
                    }
                    tmem_st16(sreg + ch * 16, pk);
                    // P goes to P V in parts of two chunks (64 keys): fewer
                    // store waits on the softmax side
                    if ((ch & 1) || ch == NC - 1) {
                        tmem_wait_st();
                        tc_fence_before_sync();
                        mbar_arrive(&parts[ch]);
                    }
                }
                const float2 l2 = __fadd2_rn(lq[0], lq[1]);
                l = l * alpha + (l2.x + l2.y);
                if (pend_kk >= 0) {
                    if (!epilogue(pend_kk, pend_off, pend_l)) {
                        failed = true;
                        break;
                    }
                    pend_kk = -1;
                }
            }
            if (failed)
                break;
            // log-sum-exp of the row's scores in natural units (m is in log2 units)
            if (lse && !me.pad)
                lse[me.offset / D] = (m + log2f(l)) * kLn2;
            if constexpr (NOB == 2) {
                pend_kk = kk;
                pend_off = me.pad ? -1 : me.offset;
                pend_l = l;
            } else if (!epilogue(kk, me.pad ? -1 : me.offset, l)) {
                failed = true;
                break;
            }
        }
        if (!failed && pend_kk >= 0)
            epilogue(pend_kk, pend_off, pend_l);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace winattn
