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
// Roles (416 threads):
//   warps 8-11  loader: cp.async gathers of Q, K, V (and the rank-r factors)
//               straight into the swizzled operand tiles of a ring of stages,
//               several items ahead; then, per item, window-local RoPE on Q and
//               K in place (fp32 registers), Q scaled by d^-1/2;
//   warp 12     MMA issuer (one thread): S = Q~ K~^T into TMEM, then
//               O = P V with P read from TMEM (the tensor core never waits for
//               P in shared memory);
//   warps 0-7   two softmax warpgroups, alternating items: each thread owns one
//               row (TMEM lane), computes max / exp / sum over its window's
//               keys only, writes P (bf16 pairs) over the consumed S columns,
//               and after O lands normalises and stores it to the token's
//               original (un-shifted) position.
// Every wait is a bounded mbarrier wait; a timeout sets a CTA-wide abort flag
// and the device status word, and every role drains and returns.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "geometry.cuh"
#include "ptx.cuh"

namespace winattn {

constexpr int kSmallThreads = 416;

template <int D, int R>
struct SmallLayout {
    static constexpr uint32_t QC = 0;                       // query content  [128][D] bf16, swizzled
    static constexpr uint32_t QB = QC + 256 * D;            // query factors  [128][R]
    static constexpr uint32_t KC = QB + 256 * R;            // key content    [128][D]
    static constexpr uint32_t KB = KC + 256 * D;            // key factors    [128][R]
    static constexpr uint32_t VO = KB + 256 * R;            // values         [128][D]
    static constexpr uint32_t CODES = VO + 256 * D;         // key mask codes u16[128]
    static constexpr uint32_t STAGE = (CODES + 256 + 1023) & ~1023u;
    static constexpr int NS = (200 * 1024 / STAGE) < 5 ? (200 * 1024 / STAGE) : 5;  // ring depth
    static constexpr int PF = NS - 1;                       // items in flight ahead of conversion
    static constexpr uint32_t TABLE = NS * STAGE;           // RoPE (cos, sin) [heads][M][D/4]
    static constexpr int kBars = 2 * NS + 9;
    static __host__ __device__ uint32_t table_bytes(int heads, int M)
    {
        return (uint32_t)(heads * M * (D / 4) * 8 + 15) & ~15u;
    }
    static __host__ __device__ uint32_t bars(int heads, int M) { return TABLE + table_bytes(heads, M); }
    static __host__ __device__ uint32_t bytes(int heads, int M) { return bars(heads, M) + kBars * 8 + 16 + 1024; }
};

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1u;
            atomicOr(&g_status_word, 1u);
            return false;
        }
    }
    return true;
}

// The same, with one verdict for the whole warp (its tcgen05 loads and stores
// are warp-collective, so the warp must leave a loop together).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag)
{
    return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag));
}

// Row `row` of a swizzled bf16 tile: rotate by R(i, j) (when table != null),
// multiply by `mul`, write back in place.
template <int D>
__device__ __forceinline__ void rotate_row_inplace(uint8_t *tile, int row, const float2 *table, int i, int j,
                                                   float mul)
{
    float x[D];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + swz_offset(row, c, 2 * D));
        x[8 * c + 0] = bf16lo(u.x); x[8 * c + 1] = bf16hi(u.x);
        x[8 * c + 2] = bf16lo(u.y); x[8 * c + 3] = bf16hi(u.y);
        x[8 * c + 4] = bf16lo(u.z); x[8 * c + 5] = bf16hi(u.z);
        x[8 * c + 6] = bf16lo(u.w); x[8 * c + 7] = bf16hi(u.w);
    }
    if (table) {
#pragma unroll
        for (int k = 0; k < D / 4; ++k) {
            const float2 ry = table[i * (D / 4) + k];
            const float a0 = x[2 * k], a1 = x[2 * k + 1];
            x[2 * k] = a0 * ry.x - a1 * ry.y;
            x[2 * k + 1] = a0 * ry.y + a1 * ry.x;
            const float2 rx = table[j * (D / 4) + k];
            const float b0 = x[D / 2 + 2 * k], b1 = x[D / 2 + 2 * k + 1];
            x[D / 2 + 2 * k] = b0 * rx.x - b1 * rx.y;
            x[D / 2 + 2 * k + 1] = b0 * rx.y + b1 * rx.x;
        }
    }
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 o;
        o.x = pack_bf16x2(x[8 * c + 0] * mul, x[8 * c + 1] * mul);
        o.y = pack_bf16x2(x[8 * c + 2] * mul, x[8 * c + 3] * mul);
        o.z = pack_bf16x2(x[8 * c + 4] * mul, x[8 * c + 5] * mul);
        o.w = pack_bf16x2(x[8 * c + 6] * mul, x[8 * c + 7] * mul);
        *reinterpret_cast<uint4 *>(tile + swz_offset(row, c, 2 * D)) = o;
    }
}

template <int D, int R>
__global__ void __launch_bounds__(kSmallThreads, 1)
    winattn_fwd_small_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                             const __nv_bfloat16 *__restrict__ v, const float *__restrict__ theta,
                             const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ out,
                             const Geometry g, const float scale)
{
    using L = SmallLayout<D, R>;
    constexpr int NS = L::NS, PF = L::PF;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    float2 *table = reinterpret_cast<float2 *>(base + L::TABLE);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::bars(g.heads, g.M));
    uint64_t *full = bars, *empty = bars + NS, *s_full = bars + 2 * NS, *p_full = s_full + 2, *o_full = p_full + 2,
             *t_free = o_full + 2, *fin = t_free + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::kBars);
    volatile uint32_t *abort_flag = tslot + 1;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int n_items = (int)g.items;
    const int first = blockIdx.x, stride = gridDim.x;
    const int count = first < n_items ? (n_items - 1 - first) / stride + 1 : 0;
    const int table_per_head = g.M * (D / 4);

    if (warp == 12) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (t == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 128);
            mbar_init(&empty[s], 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&s_full[w], 1);
            mbar_init(&p_full[w], 128);
            mbar_init(&o_full[w], 1);
            mbar_init(&t_free[w], 128);
        }
        mbar_init(fin, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (theta) {
        for (int idx = t; idx < g.heads * table_per_head; idx += blockDim.x) {
            const int h = idx / table_per_head, r = idx - h * table_per_head;
            const int c = r / (D / 4), kk = r - c * (D / 4);
            float sn, cs;
            sincosf((float)c * __ldg(theta + h * (D / 4) + kk), &sn, &cs);
            table[idx] = make_float2(cs, sn);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    if (warp >= 8 && warp < 12) {
        // ------------------------------------------------------------ loader
        const int lt = t - 256;
        constexpr int CD = D / 8, CR = R / 8;
        auto issue = [&](int kk) -> bool {
            const int s = kk % NS;
            if (kk >= NS && !wait_or_abort(&empty[s], ((kk / NS) - 1) & 1, abort_flag))
                return false;
            const Item it = decode_item_head_minor(g, first + kk * stride);
            const int pack = it.pack, h = it.h;
            uint8_t *st = base + s * L::STAGE;
            const uint32_t sst = sbase + s * L::STAGE;
#pragma unroll
            for (int i = 0; i < CD; ++i) {
                const int idx = i * 128 + lt, row = idx / CD, ch = idx % CD;
                const RowRef rr = tile_row(g, pack, 0, row);
                const uint32_t off = swz_offset(row, ch, 2 * D);
                if (rr.valid) {
                    const int64_t src = token_ref(g, rr.w, rr.p, h).offset + ch * 8;
                    cp_async16(sst + L::QC + off, q + src);
                    cp_async16(sst + L::KC + off, k + src);
                    cp_async16(sst + L::VO + off, v + src);
                } else {
                    *reinterpret_cast<uint4 *>(st + L::QC + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(st + L::KC + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(st + L::VO + off) = make_uint4(0, 0, 0, 0);
                }
            }
            if constexpr (R > 0) {
#pragma unroll
                for (int i = 0; i < CR; ++i) {
                    const int idx = i * 128 + lt, row = idx / CR, ch = idx % CR;
                    const RowRef rr = tile_row(g, pack, 0, row);
                    const uint32_t off = swz_offset(row, ch, 2 * R);
                    if (rr.valid) {
                        cp_async16(sst + L::QB + off, bias + (((int64_t)h * 2 + 0) * g.N + rr.p) * R + ch * 8);
                        cp_async16(sst + L::KB + off, bias + (((int64_t)h * 2 + 1) * g.N + rr.p) * R + ch * 8);
                    } else {
                        *reinterpret_cast<uint4 *>(st + L::QB + off) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(st + L::KB + off) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            const RowRef rr = tile_row(g, pack, 0, lt);
            uint16_t code = 0xFFFE;
            if (rr.valid)
                code = (uint16_t)((rr.slot << 2) | token_ref(g, rr.w, rr.p, h).label);
            reinterpret_cast<uint16_t *>(st + L::CODES)[lt] = code;
            return true;
        };

        // Exactly PF - 1 groups go out before the loop (empty ones when the CTA
        // has fewer items), and one more per iteration, so that waiting until
        // at most PF - 1 groups are pending always covers item kc.
        bool failed = false;
        for (int kk = 0; kk < PF - 1; ++kk) {
            if (kk < count && !failed)
                failed = !issue(kk);
            cp_async_commit();
        }
        for (int kc = 0; kc < count; ++kc) {
            const int kk = kc + PF - 1;
            if (kk < count && !failed)
                failed = !issue(kk);
            cp_async_commit();
            cp_async_wait<PF - 1>();
            // Every loader thread's copies of item kc have landed (and all
            // loader threads agree on whether to stop).
            if (named_bar_any(1, 128, failed))
                break;
            const int s = kc % NS;
            const Item it = decode_item_head_minor(g, first + kc * stride);
            const int pack = it.pack, h = it.h;
            const RowRef rr = tile_row(g, pack, 0, lt);
            if (rr.valid) {
                const TokenRef tk = token_ref(g, rr.w, rr.p, h);
                const float2 *tb = theta ? table + h * table_per_head : nullptr;
                uint8_t *st = base + s * L::STAGE;
                rotate_row_inplace<D>(st + L::QC, lt, tb, tk.i, tk.j, scale);
                if (theta)
                    rotate_row_inplace<D>(st + L::KC, lt, tb, tk.i, tk.j, 1.f);
            }
            fence_proxy_async_smem();
            mbar_arrive(&full[s]);
        }
        cp_async_wait_all();
    } else if (warp == 12) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
            auto issue_s = [&](int kc) -> bool {
                const int s = kc % NS, w = kc & 1;
                if (!wait_or_abort(&full[s], (kc / NS) & 1, abort_flag))
                    return false;
                if (kc >= 2 && !wait_or_abort(&t_free[w], ((kc - 2) >> 1) & 1, abort_flag))
                    return false;
                tc_fence_after_sync();
                const uint32_t sst = sbase + s * L::STAGE;
                const uint32_t d = tmem + w * 256;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_bf16_ss(d, smem_desc(sst + L::QC + ks * 32, 16, 16 * D, swizzle_code(2 * D)),
                                 smem_desc(sst + L::KC + ks * 32, 16, 16 * D, swizzle_code(2 * D)), kIdescS, ks > 0);
#pragma unroll
                for (int ks = 0; ks < R / 16; ++ks)
                    umma_bf16_ss(d, smem_desc(sst + L::QB + ks * 32, 16, 16 * R, swizzle_code(2 * R)),
                                 smem_desc(sst + L::KB + ks * 32, 16, 16 * R, swizzle_code(2 * R)), kIdescS, 1);
                umma_commit(&s_full[w]);
                return true;
            };
            bool ok = count > 0 ? issue_s(0) : true;
            for (int kc = 0; kc < count && ok; ++kc) {
                if (kc + 1 < count && !(ok = issue_s(kc + 1)))
                    break;
                const int s = kc % NS, w = kc & 1;
                if (!(ok = wait_or_abort(&p_full[w], (kc >> 1) & 1, abort_flag)))
                    break;
                tc_fence_after_sync();
                const uint32_t sst = sbase + s * L::STAGE;
                const uint32_t pa = tmem + w * 256;        // P: 64 columns of bf16 pairs (over S)
                const uint32_t od = tmem + w * 256 + 128;  // O: D columns
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16_ts(od, pa + ks * 8,
                                 smem_desc(sst + L::VO + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D)), kIdescPV,
                                 ks > 0);
                umma_commit(&o_full[w]);
                umma_commit(&empty[s]);
            }
            // every UMMA issued above has completed before TMEM is released
            umma_commit(fin);
            mbar_wait(fin, 0);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax + epilogue
        const int w = warp >> 2;
        const int row = t - 128 * w;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + w * 256 + lane_base;
        const uint32_t o_addr = s_addr + 128;
        const int r0 = (warp & 3) * 32;
        int c_lo = 0, c_hi = g.N < 128 ? g.N : 128;
        if (g.U > 1) {
            const int s0 = r0 / g.N, s1 = (r0 + 31) / g.N;
            c_lo = s0 * g.N;
            c_hi = (s1 + 1) * g.N < 128 ? (s1 + 1) * g.N : 128;
        }
        const int ch_lo = c_lo >> 5, ch_hi = (c_hi + 31) >> 5;
        const bool aligned = (g.N & 31) == 0;

        for (int kc = w; kc < count; kc += 2) {
            const int s = kc % NS, j = kc >> 1;
            if (!warp_wait(&full[s], (kc / NS) & 1, abort_flag))
                break;
            if (!warp_wait(&s_full[w], j & 1, abort_flag))
                break;
            tc_fence_after_sync();
            const Item it = decode_item_head_minor(g, first + kc * stride);
            const int pack = it.pack, h = it.h;
            const RowRef rr = tile_row(g, pack, 0, row);
            int qcode = 0xFFFF;
            TokenRef tk{};
            if (rr.valid) {
                tk = token_ref(g, rr.w, rr.p, h);
                qcode = (rr.slot << 2) | tk.label;
            }
            const uint16_t *codes = reinterpret_cast<const uint16_t *>(base + s * L::STAGE + L::CODES);
            // Keys need no per-element test when the row's window fills whole
            // 32-column chunks and is not wrapped.
            const bool fast = __all_sync(0xffffffffu, aligned && rr.valid && !window_wrapped(g, rr.w));

            float mx = -INFINITY;
            for (int ch = ch_lo; ch < ch_hi; ++ch) {
                float x[32];
                tmem_ld32(s_addr + ch * 32, x);
                if (fast) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        mx = fmaxf(mx, x[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (codes[ch * 32 + e] == qcode)
                            mx = fmaxf(mx, x[e]);
                }
            }
            const float m = (mx == -INFINITY) ? 0.f : mx * kLog2e;
            float l = 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t pk[16];
                if (ch >= ch_lo && ch < ch_hi) {
                    float x[32];
                    tmem_ld32(s_addr + ch * 32, x);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float p0 = fast_exp2(fmaf(x[e], kLog2e, -m));
                        float p1 = fast_exp2(fmaf(x[e + 1], kLog2e, -m));
                        if (!fast) {
                            p0 = codes[ch * 32 + e] == qcode ? p0 : 0.f;
                            p1 = codes[ch * 32 + e + 1] == qcode ? p1 : 0.f;
                        }
                        l += p0 + p1;
                        pk[e >> 1] = pack_bf16x2(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = 0u;
                }
                tmem_st16(s_addr + ch * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(&p_full[w]);

            if (!warp_wait(&o_full[w], j & 1, abort_flag))
                break;
            tc_fence_after_sync();
            float o[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c)
                tmem_ld32(o_addr + c * 32, o + c * 32);
            if (rr.valid) {
                const float inv = 1.f / l;
                uint4 *dst = reinterpret_cast<uint4 *>(out + tk.offset);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    uint4 u;
                    u.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
                    u.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                    u.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                    u.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                    dst[c] = u;
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&t_free[w]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 12) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace winattn
