// Persistent, role-pipelined forward for 16 x 16 windows (256 tokens) without
// rank-r factors, shift 0 or 8, on whole maps or maps padded by half a window,
// optionally saving each row's log-sum-exp: FlashSwin-T's M = 16 ("FLASHSWIN"
// page, section "무엇과 다른가": from M = 16 the fused kernel overtakes Swin),
// and the M = 16 point of the window-size sweep.
//
// A work item is one window-head: two 128-row query tiles (window rows 0-7 and
// 8-15) against the whole window's 256 keys.  Because all keys of a window fit
// one S of 128 x 256 fp32 (256 TMEM columns), each query tile takes one S
// MMA and one softmax pass with the exact row max: no online rescale, no key
// loop.  The roles (32 warps):
//
//   warp 28       Q/K loader: per item, the two query tiles' boxes and the
//                 window's K boxes (one, two or four per operand, by wrap
//                 kind; the cyclic shift is box coordinates) into an
//                 NSQ-stage ring;
//   warp 31       V loader: the window's V boxes into an NSV-stage ring, once
//                 the item's RoPE is done;
//   warps 0-7     two RoPE warpgroups, alternate items: rotate the item's 256
//                 query rows and 256 key rows in place in fp32, write the
//                 allowed 64-key granules of each TMEM lane quarter's rows
//                 and each epilogue warp's store record;
//   warp 29       S issuer: S = Q K^T of each query tile (M = 128, N = 256)
//                 into TMEM buffer (tile % 2); after both tiles of an item the
//                 Q/K stage goes back to the loader;
//   warp 30       P V issuer: O = P V (P from TMEM, 256 keys) into the same
//                 buffer's columns 96 onwards; after both tiles the V stage
//                 goes back;
//   warps 8-23    softmax, sixteen warps on every tile: warp (g, quarter)
//                 takes the 64-key granule g of the 32 rows of TMEM lane
//                 quarter `quarter`.  Each takes the max over its granule, the
//                 four warps of a quarter exchange it through shared memory,
//                 and each then writes exp2 (scale and log2 e in one FFMA) of
//                 its granule as packed bf16 P over S columns it has read.
//                 While they work on one buffer's tile, the other buffer's
//                 tile goes through P V, the epilogue's read of O and the next
//                 S, and four warps per SM sub-partition keep the MUFU units
//                 busy;
//   warps 24-27   epilogue: O / l as bf16 into a swizzled staging tile and TMA
//                 box stores to the original, un-shifted positions.
//
// TMEM buffer b (256 columns) over one tile: S in columns 0-255; then P of
// granule g (keys 64 g .. 64 g + 63, 32 packed columns) in columns 64 g .. 64 g
// + 31 for g = 0, 1 and 64 g + 32 .. 64 g + 63 for g = 2, 3 (the last two
// granules are exponentiated from their last chunk down, so each chunk's P
// lands on S columns already read); O in columns 96 onwards (the gap between
// granule 1's P and granule 2's, up to 64 columns).
//
// Wrap masks are structural: the key boxes of a window are its wrap-label
// regions (halves at a seam, quadrants in the corner window), each a whole
// number of 64-key granules, and a query tile never straddles the row seam.
// A map padded by half a window (H or W 8 short of a multiple of 16, as
// FlashSwin-T's 56 x 56 at M = 16) has its pad positions in the last window
// row and column, in exactly those halves: with shift 8 they are the halves
// that wrap labels already separate, without shift the last window row and
// column are split the same way.  Pad boxes load as zeros (out of the map)
// and are never stored.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fwd_large.cuh"
#include "fwd_pipe.cuh"
#include "fwd_small.cuh"
#include "geometry.cuh"
#include "ptx.cuh"
#include "waits.cuh"

namespace winattn {

constexpr int kP16Bufs = 2;  // TMEM buffers of 256 columns (one per query tile of an item)
constexpr int kP16Rope = 2;                          // RoPE warpgroups (item k goes to group k % 2)
constexpr int kP16SoftmaxWarp = 4 * kP16Rope;        // first of the sixteen softmax warps
constexpr int kP16EpiWarp = kP16SoftmaxWarp + 16;
constexpr int kP16LoadWarp = kP16EpiWarp + 4;        // Q/K loader; S issuer, P V issuer and V loader follow
constexpr int kP16Threads = (kP16LoadWarp + 4) * 32;
constexpr uint32_t kP16O = 96;                      // TMEM column of O in a buffer

// TMEM column (within a buffer) of the packed P of keys 16 c .. 16 c + 15.
__host__ __device__ constexpr uint32_t p16_pcol(int c)
{
    return (uint32_t)((c >> 2) * 64 + ((c >> 2) >= 2 ? 32 : 0) + (c & 3) * 8);
}

template <int D>
struct Pipe16Layout {
    // Q/K ring, per item: query tiles A and B [128][D], keys [256][D], swizzled
    static constexpr uint32_t QA = 0, QB = 256 * D, KT = 512 * D;
    static constexpr uint32_t QK_STAGE = 1024 * D;
    static constexpr int NSQ = D == 32 ? 4 : 2;
    // V ring, per item: values [256][D]
    static constexpr uint32_t V_STAGE = 512 * D;
    static constexpr int NSV = D == 32 ? 3 : 2;
    // metadata ring, per query tile: allowed granules of the rows of each lane
    // quarter (u32[4]; a quarter's rows lie on one side of every seam), then
    // at byte 64 the output TMA stores of each epilogue warp: int4 {x0, y0,
    // image, box shape | head column << 4} (shape 0: 16 x 2 tokens, 1: 8 x 4,
    // 2: pad positions, not stored); NM = 2 NSQ + 2 orders the writer of tile
    // k + NM after the last reader of tile k
    static constexpr int NM = 2 * NSQ + 2;
    static constexpr uint32_t MSLOT = 64 + 4 * 16;
    static constexpr uint32_t VRING = NSQ * QK_STAGE;
    static constexpr uint32_t MRING = VRING + NSV * V_STAGE;
    static constexpr int NO = D == 32 ? 2 : 1;
    static constexpr uint32_t OSTAGE = (MRING + NM * MSLOT + 1023) & ~1023u;
    static constexpr uint32_t OSUM = OSTAGE + NO * 256 * D;           // partial row sums: f32[buffer][granule][128]
    static constexpr uint32_t PMAX = OSUM + kP16Bufs * 4 * 128 * 4;   // partial row maxima: f32[buffer][granule][128]
    static constexpr uint32_t TABLE = PMAX + kP16Bufs * 4 * 128 * 4;  // RoPE (cos, sin) float4 [heads][16][D/8]
    static constexpr int kBars = 3 * NSQ + 2 * NSV + NM + 5 * kP16Bufs + 2;
    static __host__ __device__ uint32_t bars(int heads) { return TABLE + (uint32_t)heads * 16 * (D / 8) * 16; }
    static __host__ __device__ uint32_t bytes(int heads) { return bars(heads) + kBars * 8 + 16 + 1024; }
};

// Shapes this kernel serves: bf16, 16 x 16 windows, no rank-r factors, shift
// 0 or 8, a map that is a whole number of windows or padded by half a window.
// With `lse` it also writes each token's log-sum-exp (natural log of the sum
// of exp(score) over the row), as the other forward kernels do.
__host__ __device__ inline bool pipe16_ok(const Geometry &g)
{
    return g.M == 16 && g.rank == 0 && (g.shift == 0 || g.shift == 8) && (g.Hp - g.H == 0 || g.Hp - g.H == 8) &&
           (g.Wp - g.W == 0 || g.Wp - g.W == 8) && (g.d == 32 || g.d == 64);
}

// Box layout of a window: bit 0 = split into column halves (the column wrap
// seam, or pad columns), bit 1 = split into row halves (the row seam, or pad
// rows); both only in the last window column / row.
__device__ __forceinline__ int pipe16_kind(const Geometry &g, int wy, int wx)
{
    return (wx == g.nWx - 1 && (g.shift || g.Wp != g.W) ? 1 : 0) |
           (wy == g.nWy - 1 && (g.shift || g.Hp != g.H) ? 2 : 0);
}

// Tensor maps of the output stores: boxes of 16 x 2 and 8 x 4 tokens (32 rows
// of a query tile each).
struct Pipe16StoreMaps {
    CUtensorMap o16x2, o8x4;
};

// P of 16 keys: exp2(s c2 - m) of each score in x[], summed into lq and
// stored as 8 packed bf16 pairs at TMEM column `pcol`.
__device__ __forceinline__ void exp_chunk16(const uint32_t (&x)[16], float2 cc, float2 mm, float2 (&lq)[2],
                                            uint32_t pcol)
{
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
        const float2 z = __ffma2_rn(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), cc, mm);
        const float2 p = make_float2(fast_exp2(z.x), fast_exp2(z.y));
        lq[(e >> 1) & 1] = __fadd2_rn(lq[(e >> 1) & 1], p);
        pk[e >> 1] = pack_bf16x2(p.x, p.y);
    }
    tmem_st8(pcol, pk);
}

template <int D>
__global__ void __launch_bounds__(kP16Threads, 1)
    winattn_fwd_pipe16_kernel(const float *__restrict__ theta, float *__restrict__ lse, const Geometry g,
                              const float scale,
                              const __grid_constant__ WindowMaps tm_q, const __grid_constant__ WindowMaps tm_k,
                              const __grid_constant__ WindowMaps tm_v, const __grid_constant__ Pipe16StoreMaps tm_o)
{
    using L = Pipe16Layout<D>;
    constexpr int NSQ = L::NSQ, NSV = L::NSV, NM = L::NM, NB = kP16Bufs;
    // Items alternate between the two RoPE groups, so an item's Q/K stage
    // (item % NSQ) must always fall to the same group; query tiles share a
    // metadata slot every NM tiles.
    static_assert(NSQ % kP16Rope == 0, "a Q/K stage must always be consumed by the same RoPE group");
    static_assert(NM % 2 == 0 && NM == 2 * NSQ + 2, "metadata ring must order its writers after its readers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    float4 *table4 = reinterpret_cast<float4 *>(base + L::TABLE);
    float *osum = reinterpret_cast<float *>(base + L::OSUM);
    float *pmax = reinterpret_cast<float *>(base + L::PMAX);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::bars(g.heads));
    uint64_t *qk_full = bars, *ready = qk_full + NSQ, *qk_empty = ready + NSQ;
    uint64_t *v_full = qk_empty + NSQ, *v_empty = v_full + NSV, *meta_full = v_empty + NSV;
    uint64_t *s_full = meta_full + NM, *p_full = s_full + NB, *o_full = p_full + NB, *t_free = o_full + NB;
    uint64_t *max_ready = t_free + NB, *fin = max_ready + NB;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::kBars);
    volatile uint32_t *abort_flag = tslot + 1;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int n_items = (int)(g.wph * g.heads);
    const int first = blockIdx.x, stride = gridDim.x;
    const int count = first < n_items ? (n_items - 1 - first) / stride + 1 : 0;  // items of this CTA

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (t == 32) {
        for (int s = 0; s < NSQ; ++s) {
            mbar_init(&qk_full[s], 1);
            mbar_init(&ready[s], 4);       // one arrival per RoPE warp
            mbar_init(&qk_empty[s], 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int m = 0; m < NM; ++m)
            mbar_init(&meta_full[m], 4);    // one arrival per RoPE warp
        for (int b = 0; b < NB; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 16);      // one arrival per softmax warp
            mbar_init(&max_ready[b], 16);   // the same
            mbar_init(&o_full[b], 1);
            mbar_init(&t_free[b], 4);       // one arrival per epilogue warp
        }
        mbar_init(&fin[0], 1);
        mbar_init(&fin[1], 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == kP16LoadWarp && lane < 8)
        tma_prefetch_map(pick_map(lane < 4 ? tm_q : tm_k, lane & 3));
    if (warp == kP16LoadWarp + 3 && lane < 4)
        tma_prefetch_map(pick_map(tm_v, lane));
    grid_launch_dependents();
    grid_dependency_wait();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    auto window_of = [&](int w, int &b, int &wy, int &wx) {
        b = (int)g.div_img.div((uint32_t)w);
        const int rem = w - b * g.nWy * g.nWx;
        wy = (int)g.div_nWx.div((uint32_t)rem);
        wx = rem - wy * g.nWx;
    };
    auto wrap = [&](int v, int lim) { return v >= lim ? v - lim : v; };

    if (warp == kP16LoadWarp) {
        // ================================================================ Q/K loader
        // lanes 0-3: query tile A's boxes, 4-7: tile B's, 8-11: the key boxes
        int kk = 0;
        for (; kk < count; ++kk) {
            const int s = kk % NSQ;
            if (kk >= NSQ && !warp_wait(&qk_empty[s], ((kk / NSQ) - 1) & 1, abort_flag))
                break;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            int b, wy, wx;
            window_of(it.pack, b, wy, wx);
            const int kind = pipe16_kind(g, wy, wx);
            const uint32_t sst = sbase + s * L::QK_STAGE;
            if (lane == 0)
                mbar_arrive_expect_tx(&qk_full[s], (uint32_t)(L::QK_STAGE));
            __syncwarp();
            int c0 = it.h * D;
            if (lane < 8) {
                // query tile qh = rows 8 qh .. 8 qh + 7: one 16 x 8 box, or two
                // 8 x 8 boxes on the column seam
                const int qh = lane >> 2, bi = lane & 3;
                const int nbox = (kind & 1) ? 2 : 1;
                if (bi < nbox) {
                    int y0 = wrap(wy * 16 + 8 * qh + g.shift, g.Hp);
                    int x0 = wrap(wx * 16 + 8 * bi + g.shift, g.Wp);
                    debug_box(c0, x0, y0, b, D, g.heads * D, nbox == 2 ? 8 : 16, 8, g.Wp, g.Hp, g.B);
                    tma_load_4d(sst + (qh ? L::QB : L::QA) + (uint32_t)(bi * 64 * 2 * D),
                                pick_map(tm_q, nbox == 2 ? 3 : 2), c0, x0, y0, b, &qk_full[s]);
                }
            } else if (lane < 12) {
                const int bi = lane - 8;
                const int nbox = kind == 3 ? 4 : (kind ? 2 : 1);
                if (bi < nbox) {
                    const int iy0 = (kind & 2) ? ((kind == 3 ? bi >> 1 : bi) * 8) : 0;
                    const int jx0 = (kind & 1) ? ((kind == 3 ? bi & 1 : bi) * 8) : 0;
                    int y0 = wrap(wy * 16 + iy0 + g.shift, g.Hp);
                    int x0 = wrap(wx * 16 + jx0 + g.shift, g.Wp);
                    debug_box(c0, x0, y0, b, D, g.heads * D, (kind & 1) ? 8 : 16, (kind & 2) ? 8 : 16, g.Wp, g.Hp, g.B);
                    tma_load_4d(sst + L::KT + (uint32_t)(bi * (256 / nbox) * 2 * D), pick_map(tm_k, kind), c0, x0, y0,
                                b, &qk_full[s]);
                }
            }
        }
        // after an abort no consumer may take the stages armed last: wait
        // (bounded) until their loads have landed before the CTA exits
        if (*abort_flag && lane == 0)
            for (int k2 = kk > NSQ ? kk - NSQ : 0; k2 < kk; ++k2)
                mbar_wait(&qk_full[k2 % NSQ], (k2 / NSQ) & 1);
        __syncwarp();
    } else if (warp == kP16LoadWarp + 3) {
        // ================================================================ V loader
        int kk = 0;
        for (; kk < count; ++kk) {
            const int s = kk % NSV;
            // once the item's RoPE is done (its first tile's metadata)
            if (!warp_wait(&meta_full[(2 * kk) % NM], ((2 * kk) / NM) & 1, abort_flag))
                break;
            if (kk >= NSV && !warp_wait(&v_empty[s], ((kk / NSV) - 1) & 1, abort_flag))
                break;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            int b, wy, wx;
            window_of(it.pack, b, wy, wx);
            const int kind = pipe16_kind(g, wy, wx);
            if (lane == 0)
                mbar_arrive_expect_tx(&v_full[s], (uint32_t)L::V_STAGE);
            __syncwarp();
            const int nbox = kind == 3 ? 4 : (kind ? 2 : 1);
            if (lane < nbox) {
                const int bi = lane;
                const int iy0 = (kind & 2) ? ((kind == 3 ? bi >> 1 : bi) * 8) : 0;
                const int jx0 = (kind & 1) ? ((kind == 3 ? bi & 1 : bi) * 8) : 0;
                int y0 = wrap(wy * 16 + iy0 + g.shift, g.Hp);
                int x0 = wrap(wx * 16 + jx0 + g.shift, g.Wp);
                int c0 = it.h * D;
                debug_box(c0, x0, y0, b, D, g.heads * D, (kind & 1) ? 8 : 16, (kind & 2) ? 8 : 16, g.Wp, g.Hp, g.B);
                tma_load_4d(sbase + L::VRING + s * L::V_STAGE + (uint32_t)(bi * (256 / nbox) * 2 * D),
                            pick_map(tm_v, kind), c0, x0, y0, b, &v_full[s]);
            }
        }
        if (*abort_flag && lane == 0)
            for (int k2 = kk > NSV ? kk - NSV : 0; k2 < kk; ++k2)
                mbar_wait(&v_full[k2 % NSV], (k2 / NSV) & 1);
        __syncwarp();
    } else if (warp == kP16LoadWarp + 1) {
        // ================================================================ S issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, 256, false);
            int kt = 0;  // query tiles issued
            bool ok = true;
            for (int kk = 0; kk < count && ok; ++kk) {
                const int s = kk % NSQ;
                if (!(ok = wait_or_abort(&ready[s], (kk / NSQ) & 1, abort_flag)))
                    break;
                for (int qh = 0; qh < 2; ++qh, ++kt) {
                    const int b = kt % NB;
                    if (kt >= NB && !(ok = wait_or_abort(&t_free[b], ((kt / NB) - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after_sync();
                    const uint32_t sst = sbase + s * L::QK_STAGE;
                    const uint64_t qd = smem_desc(sst + (qh ? L::QB : L::QA), 16, 16 * D, swizzle_code(2 * D));
                    const uint64_t kd = smem_desc(sst + L::KT, 16, 16 * D, swizzle_code(2 * D));
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks)
                        umma_bf16_ss(tmem + b * 256, qd + 2 * ks, kd + 2 * ks, kIdescS, ks > 0);
                    umma_commit(&s_full[b]);
                }
                if (ok)
                    umma_commit(&qk_empty[s]);
            }
            if (kt > 0) {
                umma_commit(&fin[0]);
                mbar_wait(&fin[0], 0);
            }
        }
    } else if (warp == kP16LoadWarp + 2) {
        // ================================================================ P V issuer
        if (lane == 0) {
            constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
            int kt = 0;
            bool ok = true;
            for (int kk = 0; kk < count && ok; ++kk) {
                const int s = kk % NSV;
                for (int qh = 0; qh < 2; ++qh, ++kt) {
                    const int b = kt % NB;
                    if (!(ok = wait_or_abort(&p_full[b], (kt / NB) & 1, abort_flag)))
                        break;
                    if (!(ok = wait_or_abort(&v_full[s], (kk / NSV) & 1, abort_flag)))
                        break;
                    tc_fence_after_sync();
                    const uint32_t vst = sbase + L::VRING + s * L::V_STAGE;
                    // 16 keys of V are 32 D bytes: +2 D in the start-address field;
                    // P of keys 16 ks .. 16 ks + 15 in 8 packed columns
                    const uint64_t vd = smem_desc(vst, 8192, 16 * D, swizzle_code(2 * D));
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks)
                        umma_bf16_ts(tmem + b * 256 + kP16O, tmem + b * 256 + p16_pcol(ks), vd + (uint64_t)(2 * D * ks),
                                     kIdescPV, ks > 0);
                    umma_commit(&o_full[b]);
                }
                if (ok)
                    umma_commit(&v_empty[s]);
            }
            if (kt > 0) {
                umma_commit(&fin[1]);
                mbar_wait(&fin[1], 0);
            }
        }
    } else if (warp < kP16SoftmaxWarp) {
        // ================================================================ RoPE groups
        // the table only these warps read: RoPE (cos, sin) of each head,
        // table4[h][pos][k/2] = (cos k, cos k+1, sin k, sin k+1) of
        // pos * theta_h[k], even k
        if (theta) {
            float *tf = reinterpret_cast<float *>(table4);
            for (int idx = t; idx < g.heads * 16 * (D / 4); idx += 32 * kP16SoftmaxWarp) {
                const int h = idx / (16 * (D / 4)), r = idx - h * 16 * (D / 4);
                const int pos = r / (D / 4), kq = r - pos * (D / 4);
                float sn, cs;
                sincosf((float)pos * __ldg(theta + h * (D / 4) + kq), &sn, &cs);
                float *e = tf + 4 * (h * 16 * (D / 8) + pos * (D / 8) + (kq >> 1));
                e[kq & 1] = cs;
                e[2 + (kq & 1)] = sn;
            }
        }
        named_bar_sync(1, 32 * kP16SoftmaxWarp);
        const int grp = warp >> 2;
        const int row = t - 128 * grp;
        for (int kk = grp; kk < count; kk += kP16Rope) {
            const int s = kk % NSQ;
            if (!warp_wait(&qk_full[s], (kk / NSQ) & 1, abort_flag))
                break;
            uint8_t *st = base + s * L::QK_STAGE;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            int b, wy, wx;
            window_of(it.pack, b, wy, wx);
            const int kind = pipe16_kind(g, wy, wx);
            const float4 *tab = theta ? table4 + it.h * 16 * (D / 8) : nullptr;
            if (theta) {
                // window-local (i, j) of each row, in the order the boxes land
                for (int qh = 0; qh < 2; ++qh) {
                    int i, j;
                    if (kind & 1) {  // two 8 x 8 boxes: columns 0-7, then 8-15
                        i = 8 * qh + ((row & 63) >> 3);
                        j = 8 * (row >> 6) + (row & 7);
                    } else {         // one 16 x 8 box, row-major
                        i = 8 * qh + (row >> 4);
                        j = row & 15;
                    }
                    rotate_row_f2<D>(st + (qh ? L::QB : L::QA), row, tab, i, j, false, 1.f);
                }
                for (int kh = 0; kh < 2; ++kh) {
                    const int rp = kh * 128 + row;
                    int i, j;
                    if (kind == 1) {         // two 8-wide, 16-high boxes, each row-major
                        i = (rp & 127) >> 3;
                        j = 8 * (rp >> 7) + (rp & 7);
                    } else if (kind == 3) {  // four 8 x 8 quadrants, each row-major
                        i = 8 * (rp >> 7) + ((rp & 63) >> 3);
                        j = 8 * ((rp >> 6) & 1) + (rp & 7);
                    } else {                 // one 16 x 16 box, or two 16 x 8 boxes stacked
                        i = rp >> 4;
                        j = rp & 15;
                    }
                    rotate_row_f2<D>(st + L::KT, rp, tab, i, j, false, 1.f);
                }
            }
            // per query tile: this row's allowed 64-key granules, and the
            // epilogue warps' store records
            for (int qh = 0; qh < 2; ++qh) {
                uint8_t *ms = base + L::MRING + ((2 * kk + qh) % NM) * L::MSLOT;
                const int lx = (kind & 1) ? (row >> 6) : 0;  // column-seam side of this query row
                uint32_t gm;
                if (kind == 0)
                    gm = 0xF;
                else if (kind == 1)
                    gm = lx ? 0xC : 0x3;
                else if (kind == 2)
                    gm = qh ? 0xC : 0x3;
                else
                    gm = 1u << (2 * qh + lx);
                if ((row & 31) == 0) {
                    reinterpret_cast<uint32_t *>(ms)[row >> 5] = gm;
                    // the store of epilogue warp q = row / 32: 2 window rows x
                    // 16 columns, or 4 rows x 8 columns on the column seam
                    const int qw = row >> 5;
                    int iy, jx, shape;
                    if (kind & 1) {
                        iy = 8 * qh + 4 * (qw & 1);
                        jx = 8 * (qw >> 1);
                        shape = 1;
                    } else {
                        iy = 8 * qh + 2 * qw;
                        jx = 0;
                        shape = 0;
                    }
                    const int y0 = wrap(wy * 16 + iy + g.shift, g.Hp), x0 = wrap(wx * 16 + jx + g.shift, g.Wp);
                    // a box of pad positions (all of its tokens are) is not stored
                    if (y0 >= g.H || x0 >= g.W)
                        shape = 2;
                    reinterpret_cast<int4 *>(ms + 64)[qw] = make_int4(x0, y0, b, shape | (it.h * D) << 4);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ready[s]);
                mbar_arrive(&meta_full[(2 * kk) % NM]);
                mbar_arrive(&meta_full[(2 * kk + 1) % NM]);
            }
        }
    } else if (warp < kP16EpiWarp) {
        // ================================================================ softmax
        // warp (gr, quarter) takes keys [64 gr, 64 gr + 64) of the rows of lane
        // quarter `quarter`, for every tile
        const int gr = (warp - kP16SoftmaxWarp) >> 2, quarter = warp & 3, row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const float c2 = scale * kLog2e;
        const float2 cc = make_float2(c2, c2);
        const float ninf = -INFINITY;
        for (int kt = 0; kt < 2 * count; ++kt) {
            const int b = kt % NB, m = kt % NM;
            if (!warp_wait(&s_full[b], (kt / NB) & 1, abort_flag))
                break;
            if (!warp_wait(&meta_full[m], (kt / NM) & 1, abort_flag))
                break;
            tc_fence_after_sync();
            const bool on = (reinterpret_cast<const uint32_t *>(base + L::MRING + m * L::MSLOT)[quarter] >> gr) & 1u;
            const uint32_t sreg = tmem + lane_base + b * 256 + gr * 64;  // S of this granule
            const uint32_t preg = tmem + lane_base + b * 256;
            // pass 1: the max over this granule, if the rows may attend to it
            float mx = ninf;
            if (on) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    float x[32];
                    tmem_ld32(sreg + h2 * 32, x);
                    float a = fmax3(x[0], x[1], x[2]);
#pragma unroll
                    for (int e = 3; e < 31; e += 2)
                        a = fmax3(a, x[e], x[e + 1]);
                    mx = fmax3(mx, a, x[31]);
                }
            }
            // exchange with the other three granules' warps of this quarter
            float *pm = pmax + b * 4 * 128 + row;
            pm[gr * 128] = mx;
            warp_arrive(&max_ready[b]);
            if (!warp_wait(&max_ready[b], (kt / NB) & 1, abort_flag))
                break;
            mx = fmaxf(fmaxf(pm[0], pm[128]), fmaxf(pm[256], pm[384]));
            // the row max for the epilogue's log-sum-exp: granule 0's slot
            // takes the combined max (no larger than any partial it replaces
            // for a warp still reading them, so their max is unchanged)
            if (gr == 0)
                pm[0] = mx;
            const float mneg = mx == ninf ? 0.f : -mx * c2;
            const float2 mm = make_float2(mneg, mneg);
            // pass 2: P = exp2(s c2 - m) in chunks of 16 keys, granules 0 and
            // 1 from the first chunk up, 2 and 3 from the last down, so that
            // chunk c's P (8 packed columns at p16_pcol) lands on S columns of
            // this granule already read; zeros if the rows may not attend
            float2 lq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            if (on) {
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    const int c = gr < 2 ? q : 3 - q;
                    uint32_t xa[16];
                    tmem_ld16_issue(sreg + c * 16, xa);
                    tmem_wait_ld16(xa);
                    exp_chunk16(xa, cc, mm, lq, preg + p16_pcol(4 * gr + c));
                }
            } else {
                uint32_t z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    z[e] = 0u;
                tmem_st16(preg + p16_pcol(4 * gr), z);
                tmem_st16(preg + p16_pcol(4 * gr) + 16, z);
            }
            const float2 l2 = __fadd2_rn(lq[0], lq[1]);
            osum[(b * 4 + gr) * 128 + row] = l2.x + l2.y;
            tmem_wait_st();
            tc_fence_before_sync();
            warp_arrive(&p_full[b]);
        }
    } else if (warp < kP16LoadWarp) {
        // ================================================================ epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        int kt = 0;
        for (; kt < 2 * count; ++kt) {
            const int b = kt % NB, e = kt % L::NO, m = kt % NM;
            // (p_full: the row sums the softmax warps wrote before arriving)
            if (!warp_wait(&o_full[b], (kt / NB) & 1, abort_flag) ||
                !warp_wait(&p_full[b], (kt / NB) & 1, abort_flag) ||
                !warp_wait(&meta_full[m], (kt / NM) & 1, abort_flag))
                break;
            tc_fence_after_sync();
            const int4 rec = reinterpret_cast<const int4 *>(base + L::MRING + m * L::MSLOT + 64)[quarter];
            const float *os = osum + b * 4 * 128 + row;
            const float lrow = (os[0] + os[128]) + (os[256] + os[384]);
            const float inv = 1.f / lrow;
            if (lse && (rec.w & 15) != 2) {
                // this row's token: row `lane` of the warp's store box, row-major
                const int bw = (rec.w & 15) ? 8 : 16;
                const int y = rec.y + lane / bw, x = rec.x + lane % bw, h = (rec.w >> 4) / D;
                lse[(((int64_t)rec.z * g.H + y) * g.W + x) * g.heads + h] =
                    (pmax[b * 4 * 128 + row] * (scale * kLog2e) + log2f(lrow)) * kLn2;
            }
            const float2 i2 = make_float2(inv, inv);
            // this warp's staging rows have been read by its stores of tile kt - NO
            if (kt >= L::NO)
                bulk_wait_group_read<L::NO - 1>();
            __syncwarp();
            uint8_t *ost = base + L::OSTAGE + e * 256 * D;
#pragma unroll
            for (int h2 = 0; h2 < D / 32; ++h2) {
                float o[32];
                tmem_ld32(tmem + lane_base + b * 256 + kP16O + h2 * 32, o);
                if (h2 == D / 32 - 1) {
                    tc_fence_before_sync();
                    warp_arrive(&t_free[b]);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float2 f[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        f[q] = __fmul2_rn(make_float2(o[8 * c + 2 * q], o[8 * c + 2 * q + 1]), i2);
                    *reinterpret_cast<uint4 *>(ost + swz_offset(row, h2 * 4 + c, 2 * D)) =
                        make_uint4(pack_bf16x2(f[0].x, f[0].y), pack_bf16x2(f[1].x, f[1].y),
                                   pack_bf16x2(f[2].x, f[2].y), pack_bf16x2(f[3].x, f[3].y));
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && (rec.w & 15) != 2) {
                int c0 = rec.w >> 4, x0 = rec.x, y0 = rec.y, bb = rec.z;
                const int shape = rec.w & 15;
                debug_box(c0, x0, y0, bb, D, g.heads * D, shape ? 8 : 16, shape ? 4 : 2, g.W, g.H, g.B);
                tma_store_4d(shape ? &tm_o.o8x4 : &tm_o.o16x2,
                             sbase + L::OSTAGE + e * 256 * D + (uint32_t)(quarter * 32 * 2 * D), c0, x0, y0, bb);
            }
            bulk_commit_group();
        }
        bulk_wait_group<0>();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace winattn
