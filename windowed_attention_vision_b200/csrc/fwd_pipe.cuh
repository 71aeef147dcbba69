// Persistent, role-pipelined forward for 8 x 8 windows (64 tokens, two
// windows per 128-row tile) without rank-r factors and with shift 0 or 4:
// Swin's stage-1 shape at patch 4 ("FLASHSWIN" page, section "무엇과
// 다른가"), where the fused kernel has to run at memory speed.
//
// Every tile passes six roles, each working on a different tile at a time,
// so that the latencies of one (TMA arrivals, tcgen05 round trips, the long
// per-row RoPE and softmax chains) hide behind the others:
//
//   warp 20       Q/K loader: each window's Q and K head slices as one box
//                 (interior), two (a seam's row or column) or four (corner)
//                 boxes straight into the swizzled operand tiles of an
//                 NSQ-stage ring;
//   warp 23       V loader: the same boxes of V into an NSV-stage ring, issued
//                 once the tile's RoPE is done, so that V arrives about when
//                 P V needs it instead of occupying shared memory through the
//                 whole pipeline;
//   warps 0-7     two RoPE warpgroups, alternate tiles: a thread owns one
//                 tile row: it resolves the row's token (window-local (i, j)
//                 in box order, original position, wrap-label granules) and
//                 rotates its Q and K rows in place in fp32;
//   warps 21, 22  MMA issuers: S = Q K^T of each tile into TMEM buffer
//                 k % 4 as soon as its RoPE is done and the buffer is free
//                 (the commit also frees the tile's Q/K stage); O = P V as
//                 soon as its P is written and its V has landed (the commit
//                 frees the V stage).  Each issuer blocks in bounded mbarrier
//                 waits (a try_wait holds the thread in hardware), so neither
//                 spins on the issue slots others need;
//   warps 8-15    two softmax warpgroups, alternate tiles: max / exp2 / sum
//                 of a row over its own window's allowed keys, P (bf16 pairs)
//                 written over the consumed S columns;
//   warps 16-19   epilogue: O / l of each row, as bf16, into a staging tile
//                 written back with TMA stores of the same boxes the loaders
//                 read: the token's original, un-shifted position.
//
// The rings must cover the DRAM latency plus the processing latency of the
// tiles in flight, so Q/K (needed until S) and V (needed from P V only) have
// rings of their own.  Per-row metadata (wrap-label granules) lives in a ring
// of its own that outlasts the Q/K stage.  Measured per tile, the steady rate
// is set by the TMA issue rate of the SM (four box loads and two to four box
// stores per tile), not by the ring depths or any one role.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fwd_small.cuh"
#include "geometry.cuh"
#include "ptx.cuh"
#include "waits.cuh"

namespace winattn {

// One arrival per warp on a barrier that counts warps rather than threads:
// the warp barrier orders every lane's earlier writes (shared memory, and
// tcgen05 operations the caller has fenced with tcgen05.fence::before_thread_sync)
// before lane 0's release-arrive.  One arrive instead of 32 same-address
// shared-memory atomics per warp.
__device__ __forceinline__ void warp_arrive(uint64_t *bar)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        mbar_arrive(bar);
}

constexpr int kPipeRope = 2;                    // RoPE warpgroups (tile k goes to group k % 2)
constexpr int kPipeSoftmaxWarp = 4 * kPipeRope; // first softmax warp
constexpr int kPipeEpiWarp = kPipeSoftmaxWarp + 8;
constexpr int kPipeLoadWarp = kPipeEpiWarp + 4; // Q/K loader; S issuer, P V issuer and V loader follow
constexpr int kPipeThreads = (kPipeLoadWarp + 4) * 32;
constexpr int kPipeBufs = 4;  // TMEM buffers (tiles between S and the epilogue)

template <int D>
struct PipeLayout {
    // Q/K ring: query and key content [128][D] bf16 each, swizzled
    static constexpr uint32_t QC = 0, KC = 256 * D;
    static constexpr uint32_t QK_STAGE = 512 * D;
    static constexpr int NSQ = D == 32 ? 8 : 4;
    // V ring: values [128][D]
    static constexpr uint32_t V_STAGE = 256 * D;
    static constexpr int NSV = D == 32 ? 6 : 3;
    // metadata ring, per tile: allowed granules of each row, i64[128], then
    // the output TMA stores of each warp: int4[4 warps][2] = {x0, y0, image,
    // box shape | head column << 4} (box shape -1: no store)
    static constexpr int NM = NSQ + kPipeBufs;
    static constexpr uint32_t MSLOT = 128 * 8 + 8 * 16;
    static constexpr uint32_t VRING = NSQ * QK_STAGE;
    static constexpr uint32_t MRING = VRING + NSV * V_STAGE;
    // output staging for the TMA stores: [128][D] bf16, swizzled like the operands
    static constexpr int NO = D == 32 ? 2 : 1;
    static constexpr uint32_t OSTAGE = (MRING + NM * MSLOT + 1023) & ~1023u;
    static constexpr uint32_t OSUM = OSTAGE + NO * 256 * D;         // per TMEM buffer: row sum l, f32[4][128]
    static constexpr uint32_t OMAX = OSUM + kPipeBufs * 128 * 4;    // per TMEM buffer: row max (log2 units)
    static constexpr uint32_t IJTAB = OMAX + kPipeBufs * 128 * 4;   // box row order: (i << 8 | j) u16[4][64]
    static constexpr uint32_t TABLE = IJTAB + 512;                  // RoPE (cos, sin) float4 [heads][8][D/8]
    static constexpr int kBars = 3 * NSQ + 2 * NSV + NM + 4 * kPipeBufs + 2;
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
    winattn_fwd_pipe_kernel(const float *__restrict__ theta, __nv_bfloat16 *__restrict__ out,
                            float *__restrict__ lse, const Geometry g,
                            const float scale, const __grid_constant__ WindowMaps tm_q,
                            const __grid_constant__ WindowMaps tm_k, const __grid_constant__ WindowMaps tm_v,
                            const __grid_constant__ WindowMaps tm_o)
{
    using L = PipeLayout<D>;
    constexpr int NSQ = L::NSQ, NSV = L::NSV, NM = L::NM, NB = kPipeBufs;
    static_assert(NSQ >= 3 && NSV >= 2, "rings too shallow");
    // mbarrier waits test a phase's parity only, so a waiter must never reach
    // phase u + 2 of a barrier while phase u is still pending.  Tiles k and
    // k + NSQ share a Q/K stage and must fall to the same RoPE group (which
    // takes them in order); tiles k and k + NM share a metadata slot and must
    // fall to the same softmax group.  NM = NSQ + NB also orders the metadata
    // writer of tile k + NM after the last reader of tile k (S of tile
    // k + NB needs tile k's TMEM buffer back from the epilogue).
    static_assert(NSQ % kPipeRope == 0, "a Q/K stage must always be consumed by the same RoPE group");
    static_assert(NM % 2 == 0 && NM == NSQ + NB, "metadata ring must order its writers after its readers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    uint16_t *ijtab = reinterpret_cast<uint16_t *>(base + L::IJTAB);
    float2 *table = reinterpret_cast<float2 *>(base + L::TABLE);
    float *osum = reinterpret_cast<float *>(base + L::OSUM);
    float *omax = reinterpret_cast<float *>(base + L::OMAX);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::bars(g.heads));
    uint64_t *qk_full = bars, *ready = qk_full + NSQ, *qk_empty = ready + NSQ;
    uint64_t *v_full = qk_empty + NSQ, *v_empty = v_full + NSV, *meta_full = v_empty + NSV;
    uint64_t *s_full = meta_full + NM, *p_full = s_full + NB, *o_full = p_full + NB, *t_free = o_full + NB;
    uint64_t *fin = t_free + NB;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::kBars);
    volatile uint32_t *abort_flag = tslot + 1;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int n_items = (int)g.items;
    const int first = blockIdx.x, stride = gridDim.x;
    const int count = first < n_items ? (n_items - 1 - first) / stride + 1 : 0;
    constexpr int kTab = 8 * (D / 4);  // table float pairs per head: 8 positions x D/4 frequencies

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
            mbar_init(&p_full[b], 4);       // one arrival per softmax warp
            mbar_init(&o_full[b], 1);
            mbar_init(&t_free[b], 4);       // one arrival per epilogue warp
        }
        mbar_init(&fin[0], 1);
        mbar_init(&fin[1], 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    // the tensor maps (kernel parameters, not data) are fetched one per lane
    if (warp == kPipeLoadWarp && lane < 12)
        tma_prefetch_map(pick_map(lane < 4 ? tm_q : (lane < 8 ? tm_k : tm_o), lane & 3));
    if (warp == kPipeLoadWarp + 3 && lane < 4)
        tma_prefetch_map(pick_map(tm_v, lane));
    // TMEM and the barriers are set up; nothing of global memory is touched
    // before the previous kernel of the stream has completed
    grid_launch_dependents();
    grid_dependency_wait();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    // The boxes of tile k, one per loader lane (window slot, box): the
    // rolled-window origin of the box, its original coordinates and its row
    // offset in the operand tile.
    struct Box {
        bool go;
        int kind, c0, x0, y0, b;
        uint32_t roff;
    };
    auto box_of = [&](const Item &it, int nvalid) -> Box {
        Box r{};
        r.go = false;
        const int my_slot = lane >> 2, my_box = lane & 3;
        if (my_slot >= nvalid)
            return r;
        const int w = it.pack * 2 + my_slot;
        r.b = (int)g.div_img.div((uint32_t)w);
        const int rem = w - r.b * g.nWy * g.nWx;
        const int wy = (int)g.div_nWx.div((uint32_t)rem);
        const int wx = rem - wy * g.nWx;
        r.kind = window_kind(g, wy, wx);
        const int nbox = r.kind == 3 ? 4 : (r.kind ? 2 : 1);
        if (my_box >= nbox)
            return r;
        const int bi = my_box;
        const int iy0 = (r.kind & 2) ? ((r.kind == 3 ? bi >> 1 : bi) * 4) : 0;
        const int jx0 = (r.kind & 1) ? ((r.kind == 3 ? bi & 1 : bi) * 4) : 0;
        r.y0 = wy * 8 + iy0 + g.shift;
        if (r.y0 >= g.H) r.y0 -= g.H;
        r.x0 = wx * 8 + jx0 + g.shift;
        if (r.x0 >= g.W) r.x0 -= g.W;
        r.roff = (uint32_t)((my_slot * 64 + bi * (64 / nbox)) * 2 * D);
        r.c0 = it.h * D;
        r.go = true;
        debug_box(r.c0, r.x0, r.y0, r.b, D, g.heads * D, (r.kind & 1) ? 4 : 8, (r.kind & 2) ? 4 : 8, g.W, g.H, g.B);
        return r;
    };
    auto valid_windows = [&](const Item &it) -> int {
        const int64_t left = g.wph - (int64_t)it.pack * 2;
        return left < 2 ? (int)left : 2;
    };

    if (warp == kPipeLoadWarp) {
        // ================================================================ Q/K loader
        // (starts right after the CTA barrier: the first tiles' DRAM latency
        // overlaps the RoPE warps' table setup)
        int kk = 0;
        for (; kk < count; ++kk) {
            const int s = kk % NSQ;
            if (kk >= NSQ && !warp_wait(&qk_empty[s], ((kk / NSQ) - 1) & 1, abort_flag))
                break;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const int nvalid = valid_windows(it);
            const uint32_t sst = sbase + s * L::QK_STAGE;
            if (lane == 0)
                mbar_arrive_expect_tx(&qk_full[s], (uint32_t)(2 * nvalid * 64 * 2 * D));
            __syncwarp();
            const Box r = box_of(it, nvalid);
            if (r.go) {
                tma_load_4d(sst + L::QC + r.roff, pick_map(tm_q, r.kind), r.c0, r.x0, r.y0, r.b, &qk_full[s]);
                tma_load_4d(sst + L::KC + r.roff, pick_map(tm_k, r.kind), r.c0, r.x0, r.y0, r.b, &qk_full[s]);
            }
        }
        // after an abort no consumer may take the stages armed last: wait
        // (bounded) until their loads have landed before the CTA exits
        if (*abort_flag && lane == 0)
            for (int k2 = kk > NSQ ? kk - NSQ : 0; k2 < kk; ++k2)
                mbar_wait(&qk_full[k2 % NSQ], (k2 / NSQ) & 1);
        __syncwarp();
    } else if (warp == kPipeLoadWarp + 3) {
        // ================================================================ V loader
        int kk = 0;
        for (; kk < count; ++kk) {
            const int s = kk % NSV;
            // once the tile's RoPE is done, V has about the S and softmax
            // time to arrive before P V needs it
            if (!warp_wait(&meta_full[kk % NM], (kk / NM) & 1, abort_flag))
                break;
            if (kk >= NSV && !warp_wait(&v_empty[s], ((kk / NSV) - 1) & 1, abort_flag))
                break;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const int nvalid = valid_windows(it);
            const uint32_t sst = sbase + L::VRING + s * L::V_STAGE;
            if (nvalid < 2) {
                // the empty second slot of the last pack: zero value rows (its
                // P is zero, so they only have to be finite)
                uint4 *z = reinterpret_cast<uint4 *>(base + L::VRING + s * L::V_STAGE + 64 * 2 * D);
                for (int c = lane; c < 64 * 2 * D / 16; c += 32)
                    z[c] = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive_expect_tx(&v_full[s], (uint32_t)(nvalid * 64 * 2 * D));
            __syncwarp();
            const Box r = box_of(it, nvalid);
            if (r.go)
                tma_load_4d(sst + r.roff, pick_map(tm_v, r.kind), r.c0, r.x0, r.y0, r.b, &v_full[s]);
        }
        if (*abort_flag && lane == 0)
            for (int k2 = kk > NSV ? kk - NSV : 0; k2 < kk; ++k2)
                mbar_wait(&v_full[k2 % NSV], (k2 / NSV) & 1);
        __syncwarp();
    } else if (warp == kPipeLoadWarp + 1) {
        // ================================================================ S issuer
        // S = Q K^T of each tile into TMEM buffer k % 4 as soon as its RoPE is
        // done and the buffer's previous tile has left the epilogue; the
        // commit also hands the Q/K stage back to its loader.
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
            int kk = 0;
            for (; kk < count; ++kk) {
                const int s = kk % NSQ, b = kk % NB;
                if (!wait_or_abort(&ready[s], (kk / NSQ) & 1, abort_flag))
                    break;
                if (kk >= NB && !wait_or_abort(&t_free[b], ((kk / NB) - 1) & 1, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t sst = sbase + s * L::QK_STAGE;
                // descriptors built once per tile; a 16-element K step is +32
                // bytes, i.e. +2 in the 16-byte start-address field
                const uint64_t qd = smem_desc(sst + L::QC, 16, 16 * D, swizzle_code(2 * D));
                const uint64_t kd = smem_desc(sst + L::KC, 16, 16 * D, swizzle_code(2 * D));
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_bf16_ss(tmem + b * 128, qd + 2 * ks, kd + 2 * ks, kIdescS, ks > 0);
                umma_commit(&s_full[b]);
                umma_commit(&qk_empty[s]);
            }
            if (kk > 0) {
                umma_commit(&fin[0]);
                mbar_wait(&fin[0], 0);
            }
        }
    } else if (warp == kPipeLoadWarp + 2) {
        // ================================================================ P V issuer
        // O = P V of each tile once its P is written and its V has landed;
        // the commit also hands the V stage back to its loader.
        if (lane == 0) {
            constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
            int kk = 0;
            for (; kk < count; ++kk) {
                const int s = kk % NSV, b = kk % NB;
                if (!wait_or_abort(&p_full[b], (kk / NB) & 1, abort_flag))
                    break;
                if (!wait_or_abort(&v_full[s], (kk / NSV) & 1, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t vst = sbase + L::VRING + s * L::V_STAGE;
                // 16 keys of V are 32 D bytes: +2 D in the start-address field
                const uint64_t vd = smem_desc(vst, 8192, 16 * D, swizzle_code(2 * D));
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16_ts(tmem + b * 128 + 64, tmem + b * 128 + ks * 8, vd + (uint64_t)(2 * D * ks), kIdescPV,
                                 ks > 0);
                umma_commit(&o_full[b]);
                umma_commit(&v_empty[s]);
            }
            if (kk > 0) {
                umma_commit(&fin[1]);
                mbar_wait(&fin[1], 0);
            }
        }
    } else if (warp < kPipeSoftmaxWarp) {
        // ================================================================ RoPE groups
        // the tables only these warps read: RoPE (cos, sin) of each head,
        // table4[h][pos][k/2] = (cos k, cos k+1, sin k, sin k+1) of
        // pos * theta_h[k], even k; and the window-local (i, j) of each row
        // of a box of each kind
        if (theta) {
            float *tf = reinterpret_cast<float *>(table);
            for (int idx = t; idx < g.heads * kTab; idx += 32 * kPipeSoftmaxWarp) {
                const int h = idx / kTab, r = idx - h * kTab;
                const int c = r / (D / 4), kk = r - c * (D / 4);
                float sn, cs;
                sincosf((float)c * __ldg(theta + h * (D / 4) + kk), &sn, &cs);
                float *e = tf + 2 * ((h * 8 + c) * (D / 4) + (kk & ~1));
                e[kk & 1] = cs;
                e[2 + (kk & 1)] = sn;
            }
        }
        for (int idx = t; idx < 4 * 64; idx += 32 * kPipeSoftmaxWarp) {
            const int kind = idx >> 6, rp = idx & 63;
            int i, j;
            tma_row_coords(g, kind, rp, i, j);
            ijtab[idx] = (uint16_t)((i << 8) | j);
        }
        named_bar_sync(1, 32 * kPipeSoftmaxWarp);
        const int grp = warp >> 2;
        const int row = t - 128 * grp;
        const int slot = row >> 6, rp = row & 63;
        for (int kk = grp; kk < count; kk += kPipeRope) {
            const int s = kk % NSQ, m = kk % NM;
            if (!warp_wait(&qk_full[s], (kk / NSQ) & 1, abort_flag))
                break;
            uint8_t *st = base + s * L::QK_STAGE;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const int w = it.pack * 2 + slot;
            int64_t meta = -1;  // allowed 16-key granules of the row's window, -1 for no token
            uint8_t *ms = base + L::MRING + m * L::MSLOT;
            if (w < g.wph) {
                const int b = (int)g.div_img.div((uint32_t)w);
                const int rem = w - b * g.nWy * g.nWx;
                const int wy = (int)g.div_nWx.div((uint32_t)rem);
                const int wx = rem - wy * g.nWx;
                const int kind = window_kind(g, wy, wx);
                const uint32_t ij = ijtab[kind * 64 + rp];
                const int i = (int)(ij >> 8), j = (int)(ij & 0xFF);
                meta = kind == 0 ? 0xF : (kind == 3 ? 1 << (rp >> 4) : ((rp >> 5) ? 0xC : 0x3));
                if (lane < 2) {
                    // the output store(s) of the epilogue warp on this lane
                    // quarter: rows [32 h, 32 h + 32) of the window in box order
                    // are its top / bottom half (kinds 0, 2), left / right half
                    // (kind 1), or quadrants 2 h and 2 h + 1 (kind 3)
                    const int hh = (row >> 5) & 1;
                    int4 rec = make_int4(0, 0, 0, -1);
                    if (lane == 0 || kind == 3) {
                        int iy0, jx0, shape;
                        if (kind == 3) {
                            const int qd = 2 * hh + lane;
                            iy0 = (qd >> 1) * 4;
                            jx0 = (qd & 1) * 4;
                            shape = 3;
                        } else if (kind == 1) {
                            iy0 = 0;
                            jx0 = 4 * hh;
                            shape = 1;
                        } else {
                            iy0 = 4 * hh;
                            jx0 = 0;
                            shape = 2;
                        }
                        int y0 = wy * 8 + iy0 + g.shift;
                        if (y0 >= g.H) y0 -= g.H;
                        int x0 = wx * 8 + jx0 + g.shift;
                        if (x0 >= g.W) x0 -= g.W;
                        rec = make_int4(x0, y0, b, shape | (it.h * D) << 4);
                    }
                    reinterpret_cast<int4 *>(ms + 1024)[(row >> 5) * 2 + lane] = rec;
                }
                if (theta)
                    rotate_qk_rows<D>(st + L::QC, st + L::KC, row,
                                      reinterpret_cast<const float4 *>(table + it.h * kTab), i, j, false, 1.f);
            } else {
                // an empty slot of the last pack: zero rows keep its keys finite
                // (their P is zero); nothing of it is stored
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint32_t off = swz_offset(row, c, 2 * D);
                    *reinterpret_cast<uint4 *>(st + L::QC + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(st + L::KC + off) = make_uint4(0, 0, 0, 0);
                }
                if (lane < 2)
                    reinterpret_cast<int4 *>(ms + 1024)[(row >> 5) * 2 + lane] = make_int4(0, 0, 0, -1);
            }
            reinterpret_cast<int64_t *>(ms)[row] = meta;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ready[s]);
                mbar_arrive(&meta_full[m]);
            }
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
            const int b = kk % NB, m = kk % NM;
            if (!warp_wait(&s_full[b], (kk / NB) & 1, abort_flag))
                break;
            // the row's metadata (written with the tile's RoPE)
            if (!warp_wait(&meta_full[m], (kk / NM) & 1, abort_flag))
                break;
            tc_fence_after_sync();
            const int64_t meta = reinterpret_cast<const int64_t *>(base + L::MRING + m * L::MSLOT)[row];
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
            float2 lq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // two sum chains
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
                        lq[(e >> 1) & 1] = __fadd2_rn(lq[(e >> 1) & 1], p);
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
            const float2 l2 = __fadd2_rn(lq[0], lq[1]);
            osum[b * 128 + row] = l2.x + l2.y;
            omax[b * 128 + row] = -mneg;
            tmem_wait_st();
            tc_fence_before_sync();
            warp_arrive(&p_full[b]);
        }
    } else if (warp < kPipeLoadWarp) {
        // ================================================================ epilogue
        // O / l of each row, as bf16, into a staging tile laid out like the
        // operand tiles; each warp then writes its own 32 rows back with TMA
        // stores: half a window (an M x M/2 or M/2 x M box) or, in the corner
        // window, two quadrants, at the rows' original (un-shifted) position.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        int kk = 0;
        for (; kk < count; ++kk) {
            const int b = kk % NB, e = kk % L::NO, m = kk % NM;
            // the row sum was written before p_full[b] (complete: P V ran), the
            // store record with the tile's RoPE (meta_full[m])
            if (!warp_wait(&o_full[b], (kk / NB) & 1, abort_flag) ||
                !warp_wait(&p_full[b], (kk / NB) & 1, abort_flag) ||
                !warp_wait(&meta_full[m], (kk / NM) & 1, abort_flag))
                break;
            tc_fence_after_sync();
            // read before the buffer is released: the slot is rewritten only
            // after S of tile kk + 4, which needs this buffer back
            int4 rec = lane < 2 ? reinterpret_cast<const int4 *>(base + L::MRING + m * L::MSLOT + 1024)[quarter * 2 + lane]
                                : make_int4(0, 0, 0, -1);
            const float lrow = osum[b * 128 + row];
            const float inv = 1.f / lrow;
            const float2 i2 = make_float2(inv, inv);
            if (lse) {
                // the row's token from the warp's store record(s): the rows of
                // a record's box in row-major order (box widths: 8 tokens for
                // a half window of rows, 4 for a half of columns or a quadrant)
                const int4 r0 = make_int4(__shfl_sync(~0u, rec.x, 0), __shfl_sync(~0u, rec.y, 0),
                                          __shfl_sync(~0u, rec.z, 0), __shfl_sync(~0u, rec.w, 0));
                const int4 r1 = make_int4(__shfl_sync(~0u, rec.x, 1), __shfl_sync(~0u, rec.y, 1),
                                          __shfl_sync(~0u, rec.z, 1), __shfl_sync(~0u, rec.w, 1));
                const bool quad = r0.w >= 0 && (r0.w & 3) == 3;
                const int4 rr = quad && lane >= 16 ? r1 : r0;
                const int ll = quad ? (lane & 15) : lane;
                const int bw = (rr.w & 3) == 2 ? 8 : 4;
                if (rr.w >= 0) {
                    const int y = rr.y + ll / bw, x = rr.x + ll % bw, h = (rr.w >> 4) / D;
                    lse[(((int64_t)rr.z * g.H + y) * g.W + x) * g.heads + h] =
                        (omax[b * 128 + row] + log2f(lrow)) * kLn2;
                }
            }
            uint4 y[D / 8];
            // the buffer goes back to the S issuer as soon as O is in registers
#pragma unroll
            for (int h2 = 0; h2 < D / 32; ++h2) {
                float o[32];
                tmem_ld32(tmem + lane_base + b * 128 + 64 + h2 * 32, o);
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
                    y[h2 * 4 + c] = make_uint4(pack_bf16x2(f[0].x, f[0].y), pack_bf16x2(f[1].x, f[1].y),
                                               pack_bf16x2(f[2].x, f[2].y), pack_bf16x2(f[3].x, f[3].y));
                }
            }
            // this warp's staging rows have been read by its stores of tile kk - NO
            if (kk >= L::NO)
                bulk_wait_group_read<L::NO - 1>();
            __syncwarp();
            uint8_t *ost = base + L::OSTAGE + e * 256 * D;
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
                *reinterpret_cast<uint4 *>(ost + swz_offset(row, c, 2 * D)) = y[c];
            fence_proxy_async_smem();
            __syncwarp();
            if (rec.w >= 0) {
#ifdef WINATTN_DEBUG
                {
                    int c0 = rec.w >> 4, x0 = rec.x, y0 = rec.y, bb = rec.z;
                    const int shp = rec.w & 3;
                    debug_box(c0, x0, y0, bb, D, g.heads * D, shp == 2 ? 8 : 4, shp == 1 ? 8 : 4, g.W, g.H, g.B);
                    rec = make_int4(x0, y0, bb, shp | (c0 << 4));
                }
#endif
                const int shape = rec.w & 3;
                const CUtensorMap *map = shape == 3 ? &tm_o.quarter : (shape == 1 ? &tm_o.xhalf : &tm_o.yhalf);
                tma_store_4d(map, sbase + L::OSTAGE + e * 256 * D + (uint32_t)((quarter * 32 + lane * 16) * 2 * D),
                             rec.w >> 4, rec.x, rec.y, rec.z);
            }
            bulk_commit_group();
        }
        // every store has landed before the CTA exits
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
