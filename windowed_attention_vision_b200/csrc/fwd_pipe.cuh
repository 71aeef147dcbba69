// Persistent, role-pipelined forward for 8 x 8 windows (64 tokens, two
// windows per 128-row tile) without rank-r factors and with shift 0 or 4:
// Swin's stage-1 shape at patch 4 ("FLASHSWIN" page, section "무엇과
// 다른가"), where the fused kernel has to run at memory speed.
//
// Every tile passes five roles, each working on a different tile at a time,
// so that the latencies of one (TMA arrivals, tcgen05 round trips, the long
// per-row RoPE and softmax chains) hide behind the others:
//
//   warp 20       TMA loader: each window's Q, K, V head slice as one box
//                 (interior), two (a seam's row or column) or four (corner)
//                 boxes straight into the swizzled operand tiles of an
//                 NS-stage ring;
//   warps 0-7     two RoPE warpgroups, alternate tiles: a thread owns one
//                 tile row: it resolves the row's token (window-local (i, j)
//                 in box order, original position, wrap-label granules) and
//                 rotates its Q and K rows in place in fp32;
//   warps 21, 22  MMA issuers: S = Q K^T of each tile into TMEM buffer
//                 k % 4 as soon as its RoPE is done and the buffer is free
//                 (up to four tiles ahead); O = P V as soon as its P is
//                 written.  Each issuer sleeps in bounded mbarrier waits, so
//                 neither spins on the issue slots the other roles need;
//   warps 8-15    two softmax warpgroups, alternate tiles: max / exp2 / sum
//                 of a row over its own window's allowed keys, P (bf16 pairs)
//                 written over the consumed S columns;
//   warps 16-19   epilogue: O / l of each row stored (16-byte stores) to the
//                 token's original, un-shifted position.
//
// TMEM: four buffers of 128 columns: S (fp32), P over its first 64 columns,
// O over columns [64, 64 + d).  Wrap masks need no per-key test: the boxes
// of a window are exactly its wrap-label regions, so a row may see whole
// 16-key granules of its own window (all four inside, the row's box of two
// on a seam, its quadrant in the corner window); masked granules get -inf
// in the exponent.
// Every wait is bounded; a timeout sets the CTA's abort flag and the device
// status word, and every role leaves its loop at its next wait.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fwd_small.cuh"
#include "geometry.cuh"
#include "ptx.cuh"
#include "waits.cuh"

namespace winattn {

constexpr int kPipeRope = 2;                    // RoPE warpgroups (tile k goes to group k % 2)
constexpr int kPipeSoftmaxWarp = 4 * kPipeRope; // first softmax warp
constexpr int kPipeEpiWarp = kPipeSoftmaxWarp + 8;
constexpr int kPipeLoadWarp = kPipeEpiWarp + 4;
constexpr int kPipeThreads = (kPipeLoadWarp + 3) * 32;
constexpr int kPipeBufs = 4;  // TMEM buffers (tiles between S and the epilogue)

template <int D>
struct PipeLayout {
    static constexpr uint32_t QC = 0;                 // query content [128][D] bf16, swizzled
    static constexpr uint32_t KC = QC + 256 * D;      // key content
    static constexpr uint32_t VO = KC + 256 * D;      // values
    static constexpr uint32_t META = VO + 256 * D;    // per row: original offset | granule mask, i64[128]
    static constexpr uint32_t STAGE = (META + 128 * 8 + 1023) & ~1023u;
    static constexpr int NS_FIT = (int)((208u * 1024 - kSmallTableMax) / STAGE);
    static constexpr int NS = NS_FIT < 8 ? NS_FIT : 8;
    static constexpr uint32_t OMETA = NS * STAGE;                   // per TMEM buffer: row meta, i64[4][128]
    static constexpr uint32_t OSUM = OMETA + kPipeBufs * 128 * 8;   // per TMEM buffer: row sum l, f32[4][128]
    static constexpr uint32_t IJTAB = OSUM + kPipeBufs * 128 * 4;   // box row order: (i << 8 | j) u16[4][64]
    static constexpr uint32_t TABLE = IJTAB + 512;                  // RoPE (cos, sin) float4 [heads][8][D/8]
    static constexpr int kBars = 3 * NS + 4 * kPipeBufs + 2;
    static __host__ __device__ uint32_t bars(int heads) { return TABLE + ((heads * 8 * (D / 4) * 8 + 15) & ~15u); }
    static __host__ __device__ uint32_t bytes(int heads) { return bars(heads) + kBars * 8 + 16 + 1024; }
};

// Shapes this kernel serves: bf16, 8 x 8 windows, no rank-r factors, shift 0
// or 4 (so that every box is a whole number of 8-row swizzle atoms).
__host__ __device__ inline bool pipe_ok(const Geometry &g)
{
    return g.M == 8 && g.rank == 0 && (g.shift == 0 || g.shift == 4) && (g.d == 32 || g.d == 64);
}

template <int D>
__global__ void __launch_bounds__(kPipeThreads, 1)
    winattn_fwd_pipe_kernel(const float *__restrict__ theta, __nv_bfloat16 *__restrict__ out, const Geometry g,
                            const float scale, const __grid_constant__ WindowMaps tm_q,
                            const __grid_constant__ WindowMaps tm_k, const __grid_constant__ WindowMaps tm_v)
{
    using L = PipeLayout<D>;
    constexpr int NS = L::NS, NB = kPipeBufs;
    static_assert(NS >= 3, "ring too shallow");
    // mbarrier waits test a phase's parity only, so a waiter must never reach
    // phase u + 2 of a barrier before phase u has completed: tiles k and
    // k + NS share ring stage s, and the same RoPE group (which takes them in
    // order) must wait for both; likewise tiles k and k + NB share a TMEM
    // buffer and must fall to the same softmax group.
    static_assert(NS % kPipeRope == 0, "a ring stage must always be consumed by the same RoPE group");
    static_assert(NB % 2 == 0, "a TMEM buffer must always be consumed by the same softmax group");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    uint16_t *ijtab = reinterpret_cast<uint16_t *>(base + L::IJTAB);
    float2 *table = reinterpret_cast<float2 *>(base + L::TABLE);
    int64_t *ometa = reinterpret_cast<int64_t *>(base + L::OMETA);
    float *osum = reinterpret_cast<float *>(base + L::OSUM);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::bars(g.heads));
    uint64_t *full = bars, *ready = bars + NS, *empty = bars + 2 * NS;
    uint64_t *s_full = bars + 3 * NS, *p_full = s_full + NB, *o_full = p_full + NB, *t_free = o_full + NB;
    uint64_t *fin = t_free + NB;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::kBars);
    volatile uint32_t *abort_flag = tslot + 1;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int n_items = (int)g.items;
    const int first = blockIdx.x, stride = gridDim.x;
    const int count = first < n_items ? (n_items - 1 - first) / stride + 1 : 0;
    constexpr int kTab = 8 * (D / 4);  // table floats-pairs per head: 8 positions x D/4 frequencies

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (t == 32) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], 128);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 128);
            mbar_init(&o_full[b], 1);
            mbar_init(&t_free[b], 128);
        }
        mbar_init(&fin[0], 1);
        mbar_init(&fin[1], 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (theta) {
        // table4[h][pos][k/2] = (cos k, cos k+1, sin k, sin k+1) of pos * theta_h[k], even k
        float *tf = reinterpret_cast<float *>(table);
        for (int idx = t; idx < g.heads * kTab; idx += blockDim.x) {
            const int h = idx / kTab, r = idx - h * kTab;
            const int c = r / (D / 4), kk = r - c * (D / 4);
            float sn, cs;
            sincosf((float)c * __ldg(theta + h * (D / 4) + kk), &sn, &cs);
            float *e = tf + 2 * ((h * 8 + c) * (D / 4) + (kk & ~1));
            e[kk & 1] = cs;
            e[2 + (kk & 1)] = sn;
        }
    }
    for (int idx = t; idx < 4 * 64; idx += blockDim.x) {
        const int kind = idx >> 6, rp = idx & 63;
        int i, j;
        tma_row_coords(g, kind, rp, i, j);
        ijtab[idx] = (uint16_t)((i << 8) | j);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    if (warp == kPipeLoadWarp) {
        // ================================================================ TMA loader
        if (lane == 0) {
            for (int kind = 0; kind < 4; ++kind) {
                tma_prefetch_map(pick_map(tm_q, kind));
                tma_prefetch_map(pick_map(tm_k, kind));
                tma_prefetch_map(pick_map(tm_v, kind));
            }
        }
        const int my_slot = lane >> 2, my_box = lane & 3;
        for (int kk = 0; kk < count; ++kk) {
            const int s = kk % NS;
            if (kk >= NS && !warp_wait(&empty[s], ((kk / NS) - 1) & 1, abort_flag))
                break;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const uint32_t sst = sbase + s * L::STAGE;
            const int64_t left = g.wph - (int64_t)it.pack * 2;
            const int nvalid = left < 2 ? (int)left : 2;
            if (lane == 0)
                mbar_arrive_expect_tx(&full[s], (uint32_t)(3 * nvalid * 64 * 2 * D));
            __syncwarp();
            if (my_slot < nvalid) {
                const int w = it.pack * 2 + my_slot;
                const int b = (int)g.div_img.div((uint32_t)w);
                const int rem = w - b * g.nWy * g.nWx;
                const int wy = (int)g.div_nWx.div((uint32_t)rem);
                const int wx = rem - wy * g.nWx;
                const int kind = window_kind(g, wy, wx);
                const int nbox = kind == 3 ? 4 : (kind ? 2 : 1);
                if (my_box < nbox) {
                    const int bi = my_box;
                    const int iy0 = (kind & 2) ? ((kind == 3 ? bi >> 1 : bi) * 4) : 0;
                    const int jx0 = (kind & 1) ? ((kind == 3 ? bi & 1 : bi) * 4) : 0;
                    int y0 = wy * 8 + iy0 + g.shift;
                    if (y0 >= g.H) y0 -= g.H;
                    int x0 = wx * 8 + jx0 + g.shift;
                    if (x0 >= g.W) x0 -= g.W;
                    const uint32_t roff = (uint32_t)((my_slot * 64 + bi * (64 / nbox)) * 2 * D);
                    const int c0 = it.h * D;
                    tma_load_4d(sst + L::QC + roff, pick_map(tm_q, kind), c0, x0, y0, b, &full[s]);
                    tma_load_4d(sst + L::KC + roff, pick_map(tm_k, kind), c0, x0, y0, b, &full[s]);
                    tma_load_4d(sst + L::VO + roff, pick_map(tm_v, kind), c0, x0, y0, b, &full[s]);
                }
            }
        }
    } else if (warp == kPipeLoadWarp + 1) {
        // ================================================================ S issuer
        // S = Q K^T of each tile into TMEM buffer k % 4 as soon as its RoPE is
        // done and the buffer's previous tile has left the epilogue.
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
            int kk = 0;
            for (; kk < count; ++kk) {
                const int s = kk % NS, b = kk % NB;
                if (!wait_or_abort(&ready[s], (kk / NS) & 1, abort_flag))
                    break;
                if (kk >= NB && !wait_or_abort(&t_free[b], ((kk / NB) - 1) & 1, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t sst = sbase + s * L::STAGE;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_bf16_ss(tmem + b * 128, smem_desc(sst + L::QC + ks * 32, 16, 16 * D, swizzle_code(2 * D)),
                                 smem_desc(sst + L::KC + ks * 32, 16, 16 * D, swizzle_code(2 * D)), kIdescS, ks > 0);
                umma_commit(&s_full[b]);
            }
            if (kk > 0) {
                umma_commit(&fin[0]);
                mbar_wait(&fin[0], 0);
            }
        }
    } else if (warp == kPipeLoadWarp + 2) {
        // ================================================================ P V issuer
        // O = P V of each tile as soon as its P is written; the commit also
        // hands the tile's ring stage back to the loader.
        if (lane == 0) {
            constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
            int kk = 0;
            for (; kk < count; ++kk) {
                const int s = kk % NS, b = kk % NB;
                if (!wait_or_abort(&p_full[b], (kk / NB) & 1, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t vst = sbase + s * L::STAGE + L::VO;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16_ts(tmem + b * 128 + 64, tmem + b * 128 + ks * 8,
                                 smem_desc(vst + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D)), kIdescPV, ks > 0);
                umma_commit(&o_full[b]);
                umma_commit(&empty[s]);
            }
            if (kk > 0) {
                umma_commit(&fin[1]);
                mbar_wait(&fin[1], 0);
            }
        }
    } else if (warp < kPipeSoftmaxWarp) {
        // ================================================================ RoPE groups
        const int grp = warp >> 2;
        const int row = t - 128 * grp;
        const int slot = row >> 6, rp = row & 63;
        for (int kk = grp; kk < count; kk += kPipeRope) {
            const int s = kk % NS;
            if (!warp_wait(&full[s], (kk / NS) & 1, abort_flag))
                break;
            uint8_t *st = base + s * L::STAGE;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const int w = it.pack * 2 + slot;
            int64_t meta = -1;
            if (w < g.wph) {
                const int b = (int)g.div_img.div((uint32_t)w);
                const int rem = w - b * g.nWy * g.nWx;
                const int wy = (int)g.div_nWx.div((uint32_t)rem);
                const int wx = rem - wy * g.nWx;
                const int kind = window_kind(g, wy, wx);
                const uint32_t ij = ijtab[kind * 64 + rp];
                const int i = (int)(ij >> 8), j = (int)(ij & 0xFF);
                int y = wy * 8 + i + g.shift;
                if (y >= g.H) y -= g.H;
                int x = wx * 8 + j + g.shift;
                if (x >= g.W) x -= g.W;
                const int64_t off = ((((int64_t)b * g.H + y) * g.W + x) * g.heads + it.h) * D;
                const uint32_t gmask = kind == 0 ? 0xFu : (kind == 3 ? 1u << (rp >> 4) : ((rp >> 5) ? 0xCu : 0x3u));
                meta = off | (int64_t)gmask;
                if (theta)
                    rotate_qk_rows<D>(st + L::QC, st + L::KC, row,
                                      reinterpret_cast<const float4 *>(table + it.h * kTab), i, j, false, 1.f);
            } else {
                // an empty slot of the last pack: zero rows keep its keys and
                // values finite (their P is zero)
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint32_t off = swz_offset(row, c, 2 * D);
                    *reinterpret_cast<uint4 *>(st + L::QC + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(st + L::KC + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(st + L::VO + off) = make_uint4(0, 0, 0, 0);
                }
            }
            reinterpret_cast<int64_t *>(st + L::META)[row] = meta;
            fence_proxy_async_smem();
            mbar_arrive(&ready[s]);
        }
    } else if (warp < kPipeEpiWarp) {
        // ================================================================ softmax groups
        const int grp = (warp - kPipeSoftmaxWarp) >> 2;
        const int row = t - 32 * kPipeSoftmaxWarp - 128 * grp;
        const int slot = row >> 6;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        // scores in log2 units, d^-1/2 folded into the exponent
        const float c2 = scale * kLog2e;
        const float2 cc = make_float2(c2, c2);
        const float ninf = -INFINITY;
        for (int kk = grp; kk < count; kk += 2) {
            const int s = kk % NS, b = kk % NB;
            if (!warp_wait(&s_full[b], (kk / NB) & 1, abort_flag))
                break;
            // the row's meta was written before ready[s] (complete: S was issued)
            if (!warp_wait(&ready[s], (kk / NS) & 1, abort_flag))
                break;
            tc_fence_after_sync();
            const int64_t meta = reinterpret_cast<const int64_t *>(base + s * L::STAGE + L::META)[row];
            const uint32_t gmask = meta < 0 ? 0u : (uint32_t)(meta & 15);
            const uint32_t sreg = tmem + lane_base + b * 128 + slot * 64;  // this row's window: 64 S columns
            // pass 1: granule maxima
            float gm[4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float x[32];
                tmem_ld32(sreg + h2 * 32, x);
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const float *xg = x + 16 * q2;
                    float a = fmax3(xg[0], xg[1], xg[2]);
#pragma unroll
                    for (int e = 3; e < 15; e += 2)
                        a = fmax3(a, xg[e], xg[e + 1]);
                    gm[2 * h2 + q2] = fmaxf(a, xg[15]);
                }
            }
            const float mx = fmaxf(fmax3((gmask & 1u) ? gm[0] : ninf, (gmask & 2u) ? gm[1] : ninf,
                                         (gmask & 4u) ? gm[2] : ninf),
                                   (gmask & 8u) ? gm[3] : ninf);
            const float mneg = mx == ninf ? 0.f : -mx * c2;
            // pass 2: P = exp2(s c2 - m), masked granules -> 0, over the S columns just read
            float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float x[32];
                tmem_ld32(sreg + h2 * 32, x);
                uint32_t pk[16];
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const float bq = ((gmask >> (2 * h2 + q2)) & 1u) ? mneg : ninf;
                    const float2 bb = make_float2(bq, bq);
#pragma unroll
                    for (int e = 16 * q2; e < 16 * q2 + 16; e += 2) {
                        const float2 z = __ffma2_rn(make_float2(x[e], x[e + 1]), cc, bb);
                        const float2 p = make_float2(fast_exp2(z.x), fast_exp2(z.y));
                        l2 = __fadd2_rn(l2, p);
                        pk[e >> 1] = pack_bf16x2(p.x, p.y);
                    }
                }
                // P of this row's window: packed columns [slot*32, slot*32 + 32) of the buffer
                tmem_st16(tmem + lane_base + b * 128 + slot * 32 + h2 * 16, pk);
            }
            uint32_t zero[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                zero[e] = 0u;
            // the other window's keys contribute nothing to this row
            tmem_st16(tmem + lane_base + b * 128 + (1 - slot) * 32, zero);
            tmem_st16(tmem + lane_base + b * 128 + (1 - slot) * 32 + 16, zero);
            ometa[b * 128 + row] = meta;
            osum[b * 128 + row] = l2.x + l2.y;
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(&p_full[b]);
        }
    } else if (warp < kPipeLoadWarp) {
        // ================================================================ epilogue
        const int row = t - 32 * kPipeEpiWarp;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        for (int kk = 0; kk < count; ++kk) {
            const int b = kk % NB;
            if (!warp_wait(&o_full[b], (kk / NB) & 1, abort_flag))
                break;
            // row meta and sum were written before p_full[b] (complete: P V ran)
            if (!warp_wait(&p_full[b], (kk / NB) & 1, abort_flag))
                break;
            tc_fence_after_sync();
            const int64_t meta = ometa[b * 128 + row];
            const float inv = 1.f / osum[b * 128 + row];
            const float2 i2 = make_float2(inv, inv);
            // normalise 32 columns of O and store them (16-byte stores)
            auto store32 = [&](const float *o, int h2) {
                if (meta < 0)
                    return;
                uint4 *dst = reinterpret_cast<uint4 *>(out + (meta & ~(int64_t)15)) + h2 * 4;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
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
            };
            // the buffer goes back to the S issuer as soon as the last O
            // columns are in registers, before the stores
            float o[32];
            tmem_ld32(tmem + lane_base + b * 128 + 64, o);
            if constexpr (D == 32) {
                tc_fence_before_sync();
                mbar_arrive(&t_free[b]);
                store32(o, 0);
            } else {
                store32(o, 0);
                tmem_ld32(tmem + lane_base + b * 128 + 96, o);
                tc_fence_before_sync();
                mbar_arrive(&t_free[b]);
                store32(o, 1);
            }
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
