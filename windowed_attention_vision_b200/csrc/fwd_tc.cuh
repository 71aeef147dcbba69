// bf16 window-attention forward on the sm_100a tensor cores (tcgen05 UMMA,
// accumulators in TMEM).
//
// One CTA of 128 threads owns one 128-row query tile; thread t owns row t
// (TMEM lane t).  Per key tile:
//   1. gather: each thread loads one key token and one value token of the
//      window straight from the B x H x W x (heads*d) map (cyclic shift by
//      index), applies window-local 2D RoPE to the key in fp32 registers,
//      rounds to bf16 and stores K, V (and the rank-r key factors w) into
//      swizzled shared-memory operand tiles;
//   2. S = Q~ K~^T: one thread issues d/16 (+ r/16) UMMAs 128x128x16 into TMEM;
//   3. online softmax: each thread reads its S row from TMEM, masks
//      (wrap labels, packed-window blocks, ragged tails), keeps the running
//      max / sum in fp32 and writes P (bf16) into a swizzled tile;
//   4. O_tile = P V: eight UMMAs 128 x d x 16 into TMEM (the S columns, now
//      free), added to the fp32 register accumulator after rescaling.
// The query tile is gathered and rotated the same way once per CTA, scaled by
// d^-1/2 before rounding (the rank-r query factors u stay unscaled, so
// S = d^-1/2 q.k + u.w in one dot product, as the RIB page's concatenation
// [Qc, Qp][Kc, Kp]^T = Qc Kc^T + Qp Kp^T has it).
//
// Sources: "FLASHSWIN" page, section "어떻게 동작하나" (fused IO-aware kernel,
// online softmax, N x N never stored, window-local RoPE, additive wrap mask)
// and section "전제와 한계" (bf16 Q/K/V, RoPE in fp32, fp32 softmax);
// "Rank-Factorized Implicit Neural Bias" page, section 2.1.
//
// SPARSE instantiation: the gated residual of "HSMLA: Hierarchical Softmax
// Multi-scale Linear Attention for Efficient Vision Transformers" (section
// 2, Two-Path Residual Kernel).  Work items walk a list of gated windows
// only; next to S = Q~ K~^T each key tile also gives L = relu(Q) relu(K)^T
// (raw rows, a second UMMA into TMEM), masked like S, which weighs V in a
// second P V into the O_lin-local accumulator; the epilogue adds
// O_local - O_lin-local to the global linear output already in `out`.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "geometry.cuh"
#include "ptx.cuh"

namespace winattn {

template <int D, int R, bool SPARSE = false>
struct TcLayout {
    static constexpr uint32_t QC = 0;                       // query content  [128][D]  bf16
    static constexpr uint32_t QB = QC + 256 * D;            // query factors  [128][R]  bf16
    static constexpr uint32_t KC = QB + 256 * R;            // key content    [128][D]
    static constexpr uint32_t KB = KC + 256 * D;            // key factors    [128][R]
    static constexpr uint32_t VO = KB + 256 * R;            // values         [128][D]
    static constexpr uint32_t PO = VO + 256 * D;            // probabilities  2 x [128][64]
    // SPARSE only: relu(q), relu(k) of the raw rows and the linear weights
    static constexpr uint32_t QL = PO + 32768;              // [128][D]
    static constexpr uint32_t KL = QL + (SPARSE ? 256 * D : 0);
    static constexpr uint32_t LO = (KL + (SPARSE ? 256 * D : 0) + 1023) & ~1023u;  // 2 x [128][64]
    static constexpr uint32_t TB = LO + (SPARSE ? 32768 : 0);  // RoPE table [M][D/4] float2
    static __host__ __device__ uint32_t table_bytes(int M) { return (uint32_t)((M * (D / 4) * 8 + 15) & ~15); }
    static __host__ __device__ uint32_t codes(int M) { return TB + table_bytes(M); }   // [128] u16
    static __host__ __device__ uint32_t bar(int M) { return codes(M) + 256; }          // u64
    static __host__ __device__ uint32_t tslot(int M) { return bar(M) + 8; }            // u32
    static __host__ __device__ uint32_t bytes(int M) { return tslot(M) + 16 + 1024; }  // + alignment slack
};

// Gather one d-vector (bf16), rotate it by R(i, j) in fp32, multiply by `mul`,
// round to bf16 and store it as row `row` of a swizzled K-major tile.
template <int D>
__device__ __forceinline__ void gather_rotate_store(const __nv_bfloat16 *__restrict__ src, const float2 *table,
                                                   int i, int j, float mul, uint8_t *tile, int row)
{
    float x[D];
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 u = __ldg(s4 + c);
        x[8 * c + 0] = bf16lo(u.x); x[8 * c + 1] = bf16hi(u.x);
        x[8 * c + 2] = bf16lo(u.y); x[8 * c + 3] = bf16hi(u.y);
        x[8 * c + 4] = bf16lo(u.z); x[8 * c + 5] = bf16hi(u.z);
        x[8 * c + 6] = bf16lo(u.w); x[8 * c + 7] = bf16hi(u.w);
    }
    if (table) {
#pragma unroll
        for (int k = 0; k < D / 4; ++k) {
            const float2 ry = table[i * (D / 4) + k];   // (cos, sin) of i * theta_k
            const float a0 = x[2 * k], a1 = x[2 * k + 1];
            x[2 * k] = a0 * ry.x - a1 * ry.y;
            x[2 * k + 1] = a0 * ry.y + a1 * ry.x;
            const float2 rx = table[j * (D / 4) + k];   // (cos, sin) of j * theta_k
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

// Copy COLS bf16 values unchanged into row `row` of a swizzled tile.
template <int COLS>
__device__ __forceinline__ void copy_row(const __nv_bfloat16 *__restrict__ src, uint8_t *tile, int row)
{
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < COLS / 8; ++c)
        *reinterpret_cast<uint4 *>(tile + swz_offset(row, c, 2 * COLS)) = __ldg(s4 + c);
}

template <int COLS>
__device__ __forceinline__ void zero_row(uint8_t *tile, int row)
{
#pragma unroll
    for (int c = 0; c < COLS / 8; ++c)
        *reinterpret_cast<uint4 *>(tile + swz_offset(row, c, 2 * COLS)) = make_uint4(0, 0, 0, 0);
}

// 8 consecutive 32-bit columns of this thread's TMEM lane, waited on.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v)
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = __uint_as_float(r[i]);
}

// relu of a bf16 row, copied into row `row` of a swizzled tile
template <int D>
__device__ __forceinline__ void relu_row(const __nv_bfloat16 *__restrict__ src, uint8_t *tile, int row)
{
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 u = __ldg(s4 + c);
        uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // clear each bf16 half whose sign bit is set (-0 and negatives -> +0)
            const uint32_t x = w[e];
            w[e] = ((x & 0x8000u) ? 0u : (x & 0xFFFFu)) | ((x & 0x80000000u) ? 0u : (x & 0xFFFF0000u));
        }
        *reinterpret_cast<uint4 *>(tile + swz_offset(row, c, 2 * D)) = u;
    }
}

// Window of list position `li` (SPARSE), or -1 past the list.
__device__ __forceinline__ int listed_window(const int32_t *__restrict__ windows, int n_windows, int li)
{
    return li < n_windows ? __ldg(windows + li) : -1;
}

template <int D, int R, bool SPARSE = false>
__global__ void __launch_bounds__(128, 1)
    winattn_fwd_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                          const __nv_bfloat16 *__restrict__ v, const float *__restrict__ theta,
                          const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ out,
                          float *__restrict__ lse, const Geometry g, const float scale,
                          const int32_t *__restrict__ windows = nullptr, int n_windows = 0)
{
    using L = TcLayout<D, R, SPARSE>;
    extern __shared__ uint8_t smem_raw[];
    // Operand tiles need 1024-byte alignment of their shared-memory address.
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    float2 *table = reinterpret_cast<float2 *>(base + L::TB);
    uint16_t *codes = reinterpret_cast<uint16_t *>(base + L::codes(g.M));
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + L::bar(g.M));
    uint32_t *tslot = reinterpret_cast<uint32_t *>(base + L::tslot(g.M));

    const int t = threadIdx.x;
    const int warp = t >> 5;
    // SPARSE: L = relu(Q) relu(K)^T in columns [128, 256); the linear-local
    // P V accumulates over the key tiles from column 256 (no rescaling)
    constexpr uint32_t kTmemCols = SPARSE ? 512 : 128;

    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    if (t == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    Item it;
    if constexpr (SPARSE) {
        // items: heads x ceil(n_windows / U) list packs x query tiles
        const int packs = (n_windows + g.U - 1) / g.U;
        const int item = blockIdx.x;
        it.tile = item % g.n_tiles;
        const int rest = item / g.n_tiles;
        it.pack = rest % packs;
        it.h = rest / packs;
    } else {
        it = decode_item(g, blockIdx.x);
    }
    // tile row -> window: the list entry of the row's pack position (SPARSE)
    auto row_of = [&](int tile, int row) {
        RowRef r = tile_row(g, it.pack, tile, row);
        if constexpr (SPARSE) {
            const int li = g.U > 1 ? it.pack * g.U + r.slot : it.pack;
            const int w = g.U > 1 ? (r.slot < g.U ? listed_window(windows, n_windows, li) : -1)
                                  : listed_window(windows, n_windows, li);
            r.valid = w >= 0 && (g.U > 1 || r.p < g.N);
            r.w = w < 0 ? 0 : w;
        }
        return r;
    };
    if (theta) {
        for (int idx = t; idx < g.M * (D / 4); idx += blockDim.x) {
            const int c = idx / (D / 4), kk = idx - c * (D / 4);
            float sn, cs;
            sincosf((float)c * __ldg(theta + it.h * (D / 4) + kk), &sn, &cs);
            table[idx] = make_float2(cs, sn);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t tmem_row = tmem + ((uint32_t)(warp * 32) << 16);
    const float2 *tab = theta ? table : nullptr;

    // ---- query row t
    const RowRef qr = row_of(it.tile, t);
    int qcode = 0xFFFF;  // matches no key code
    const TokenRef qtk = qr.valid ? token_ref(g, qr.w, qr.p, it.h) : TokenRef{};
    const bool qreal = qr.valid && !qtk.pad;  // a pad row of a padded grid has no output
    if (qreal) {
        const TokenRef &tk = qtk;
        qcode = (qr.slot << 2) | tk.label;
        gather_rotate_store<D>(q + tk.offset, tab, tk.i, tk.j, scale, base + L::QC, t);
        if constexpr (R > 0)
            copy_row<R>(bias + (((int64_t)it.h * 2 + 0) * g.N + qr.p) * R, base + L::QB, t);
        if constexpr (SPARSE)
            relu_row<D>(q + tk.offset, base + L::QL, t);
    } else {
        zero_row<D>(base + L::QC, t);
        if constexpr (R > 0)
            zero_row<R>(base + L::QB, t);
        if constexpr (SPARSE)
            zero_row<D>(base + L::QL, t);
    }

    constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);

    float m = -INFINITY, l = 0.f;
    float o[D];
#pragma unroll
    for (int e = 0; e < D; ++e)
        o[e] = 0.f;
    float ll = 0.f;  // SPARSE: the linear-local weight sum
    uint32_t phase = 0;
    bool ok = true;

    for (int kv = 0; kv < g.n_tiles; ++kv) {
        // ---- 1. gather K (rotated), w, V for key row t
        const RowRef kr = row_of(kv, t);
        uint16_t code = 0xFFFE;
        const TokenRef tk = kr.valid ? token_ref(g, kr.w, kr.p, it.h) : TokenRef{};
        if (kr.valid && !tk.pad) {
            code = (uint16_t)((kr.slot << 2) | tk.label);
            gather_rotate_store<D>(k + tk.offset, tab, tk.i, tk.j, 1.f, base + L::KC, t);
            if constexpr (R > 0)
                copy_row<R>(bias + (((int64_t)it.h * 2 + 1) * g.N + kr.p) * R, base + L::KB, t);
            copy_row<D>(v + tk.offset, base + L::VO, t);
            if constexpr (SPARSE)
                relu_row<D>(k + tk.offset, base + L::KL, t);
        } else {
            zero_row<D>(base + L::KC, t);
            if constexpr (R > 0)
                zero_row<R>(base + L::KB, t);
            zero_row<D>(base + L::VO, t);
            if constexpr (SPARSE)
                zero_row<D>(base + L::KL, t);
        }
        codes[t] = code;
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- 2. S = Q~ K~^T
        if (t == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t a = smem_desc(sbase + L::QC + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                const uint64_t b = smem_desc(sbase + L::KC + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                umma_bf16_ss(tmem, a, b, kIdescS, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < R / 16; ++ks) {
                const uint64_t a = smem_desc(sbase + L::QB + ks * 32, 16, 16 * R, swizzle_code(2 * R));
                const uint64_t b = smem_desc(sbase + L::KB + ks * 32, 16, 16 * R, swizzle_code(2 * R));
                umma_bf16_ss(tmem, a, b, kIdescS, 1);
            }
            if constexpr (SPARSE) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t a = smem_desc(sbase + L::QL + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                    const uint64_t b = smem_desc(sbase + L::KL + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                    umma_bf16_ss(tmem + 128, a, b, kIdescS, ks > 0);
                }
            }
            umma_commit(bar);
        }
        const bool s_done = mbar_wait(bar, phase);
        phase ^= 1;
        if (__syncthreads_or(!s_done)) {
            ok = false;
            break;
        }
        tc_fence_after_sync();

        // ---- 3. online softmax on row t
        float s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            tmem_ld32(tmem_row + c * 32, s + c * 32);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
            if (codes[c] != qcode)
                s[c] = -INFINITY;
            mx = fmaxf(mx, s[c]);
        }
        const float m_new = fmaxf(m, mx * kLog2e);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = fast_exp2(m - m_use);
        float rs = 0.f;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
            float p[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                p[e] = fast_exp2(fmaf(s[8 * ch + e], kLog2e, -m_use));
                rs += p[e];
            }
            uint4 pk;
            pk.x = pack_bf16x2(p[0], p[1]);
            pk.y = pack_bf16x2(p[2], p[3]);
            pk.z = pack_bf16x2(p[4], p[5]);
            pk.w = pack_bf16x2(p[6], p[7]);
            *reinterpret_cast<uint4 *>(base + L::PO + (ch >> 3) * 16384 + swz_offset(t, ch & 7, 128)) = pk;
        }
        l = l * alpha + rs;
        m = m_new;
        if constexpr (SPARSE) {
            // linear weights of the allowed keys, unnormalised (relu rows: >= 0)
#pragma unroll 1
            for (int ch = 0; ch < 16; ++ch) {
                float sl[8];
                tmem_ld8(tmem_row + 128 + ch * 8, sl);
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = codes[8 * ch + e] == qcode ? sl[e] : 0.f;
                    ll += p[e];
                }
                uint4 pk;
                pk.x = pack_bf16x2(p[0], p[1]);
                pk.y = pack_bf16x2(p[2], p[3]);
                pk.z = pack_bf16x2(p[4], p[5]);
                pk.w = pack_bf16x2(p[6], p[7]);
                *reinterpret_cast<uint4 *>(base + L::LO + (ch >> 3) * 16384 + swz_offset(t, ch & 7, 128)) = pk;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- 4. O_tile = P V  (into the S columns)
        if (t == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = smem_desc(sbase + L::PO + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2);
                const uint64_t b = smem_desc(sbase + L::VO + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D));
                umma_bf16_ss(tmem, a, b, kIdescPV, ks > 0);
                if constexpr (SPARSE) {
                    const uint64_t al = smem_desc(sbase + L::LO + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2);
                    umma_bf16_ss(tmem + 256, al, b, kIdescPV, kv > 0 || ks > 0);
                }
            }
            umma_commit(bar);
        }
        const bool o_done = mbar_wait(bar, phase);
        phase ^= 1;
        if (__syncthreads_or(!o_done)) {
            ok = false;
            break;
        }
        tc_fence_after_sync();
        float ot[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
            tmem_ld32(tmem_row + c * 32, ot + c * 32);
#pragma unroll
        for (int e = 0; e < D; ++e)
            o[e] = fmaf(o[e], alpha, ot[e]);

        tc_fence_before_sync();
        __syncthreads();
    }

    // SPARSE: the linear-local P V of this row, read by every lane (TMEM loads
    // are warp-collective: never under a per-row condition)
    float olr[SPARSE ? D : 1];
    if constexpr (SPARSE) {
        if (ok) {
            tc_fence_after_sync();
#pragma unroll
            for (int c = 0; c < D / 32; ++c)
                tmem_ld32(tmem_row + 256 + c * 32, olr + c * 32);
        }
    }

    // ---- normalise and write back to the original (un-shifted) position
    if (ok && qreal) {
        const TokenRef &tk = qtk;
        const float inv = 1.f / l;
        // log-sum-exp of the row's scores in natural units (m is in log2 units)
        if (lse)
            lse[tk.offset / D] = (m + log2f(l)) * kLn2;
        uint4 *dst = reinterpret_cast<uint4 *>(out + tk.offset);
        if constexpr (SPARSE) {
            // out = O_lin (already there) + O_local - O_lin-local
            const float linv = ll > 0.f ? 1.f / ll : 0.f;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 u = dst[c];
                const float base_in[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y),
                                          bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    o[8 * c + e] = base_in[e] + o[8 * c + e] * inv - olr[8 * c + e] * linv;
            }
        }
        if constexpr (SPARSE) {
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
                dst[c] = make_uint4(pack_bf16x2(o[8 * c + 0], o[8 * c + 1]), pack_bf16x2(o[8 * c + 2], o[8 * c + 3]),
                                    pack_bf16x2(o[8 * c + 4], o[8 * c + 5]), pack_bf16x2(o[8 * c + 6], o[8 * c + 7]));
        } else {
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                uint4 w;
                w.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
                w.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                w.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                w.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                dst[c] = w;
            }
        }
    }
    if (!ok) {
        if (t == 0) {
            atomicOr(&g_status_word, 1u);
            // Give an MMA that may still be in flight one more bounded chance
            // to land before its TMEM is released.
            mbar_wait(bar, phase);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace winattn
