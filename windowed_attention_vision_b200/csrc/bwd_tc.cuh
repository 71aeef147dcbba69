// Backward pass of the fused window attention on the sm_100a tensor cores:
// the gradients of a loss with respect to q, k, v, the RoPE frequencies theta
// and the rank-r bias table, given dO and the per-row log-sum-exp the forward
// saved.  The FLASHSWIN page trains the model (section "무엇과 다른가": the
// score matrices and their gradients were what kept windows small in
// training) with learned theta = exp(omega) (section "어떻게 동작하나"); like
// the forward, no N x N matrix is ever stored: P is recomputed per tile as
// exp(z - lse).
//
// One CTA of 256 threads owns one 128-row key tile of a window (or of a pack
// of small windows); two threads own key row t (see the kernel).  Per
// 128-row query tile of the same window:
//   1. gather: query row t rotated by window-local 2D RoPE in fp32, scaled by
//      d^-1/2 and rounded to bf16 (with its factors u unscaled), dO row t,
//      D_t = dO_t . O_t and the saved log-sum-exp;
//   2. S^T = K~ Q~^T and dP^T = V dO^T on tcgen05 into TMEM (key rows are
//      TMEM lanes);
//   3. per key row: P^T = exp(z - lse) over the allowed queries (same window,
//      same wrap label, real tokens), dS^T = P^T (dP^T - D), both as bf16
//      into shared-memory operand tiles;
//   4. dV += P^T dO, dK~ += dS^T Q~ (dO, Q~ read MN-major), and
//      dQ~ = dS K~ (dS^T read MN-major as the A operand, K~ MN-major);
//   5. dQ~: when the window is a single tile, finalised here (scale,
//      R(-i, -j), theta gradient); otherwise added with fp32 reductions into
//      a workspace that winattn_bwd_finalize_kernel finalises.
// After the last query tile: dV and dK~ -> dK = R(-i, -j) dK~, and the key
// side of the theta gradient; the bias-table gradients (du, dw) go to fp32
// reductions straight away.
//
// Gradient rules (the oracle's backward states them the same way): with
// S = d^-1/2 (Rq).(Rk) + u.w and dS = P o (dP - rowsum(P o dP)),
// rowsum(P o dP) = dO . O;  d(Rq) = d^-1/2 dS (Rk), d(Rk) = d^-1/2 dS^T (Rq),
// du = dS w, dw = dS^T u;  dq = R(-i, -j) d(Rq);  and d/dtheta_k of a pair
// turned by i theta_k is i (dx~1 x~0 - dx~0 x~1).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fwd_tc.cuh"
#include "geometry.cuh"
#include "ptx.cuh"

namespace winattn {

template <int D, int R>
struct BwdLayout {
    static constexpr uint32_t KT = 0;                     // key content      [128][D] bf16 (rotated)
    static constexpr uint32_t KB = KT + 256 * D;          // key factors w    [128][R]
    static constexpr uint32_t VT = KB + 256 * R;          // values           [128][D]
    static constexpr uint32_t QT = VT + 256 * D;          // query content    [128][D] (rotated, scaled)
    static constexpr uint32_t QB = QT + 256 * D;          // query factors u  [128][R]
    static constexpr uint32_t OT = QB + 256 * R;          // dO               [128][D]
    static constexpr uint32_t PT = (OT + 256 * D + 1023) & ~1023u;  // P^T  2 x [128 keys][64 queries]
    static constexpr uint32_t DS = PT + 32768;            // dS^T             2 x [128][64]
    static constexpr uint32_t QI = DS + 32768;            // per query row: lse (log2 units), D, code
    static constexpr uint32_t TB = QI + 128 * 12;         // RoPE table [M][D/4] float2
    static __host__ __device__ uint32_t table_bytes(int M) { return (uint32_t)((M * (D / 4) * 8 + 15) & ~15); }
    static __host__ __device__ uint32_t red(int M) { return TB + table_bytes(M); }            // f32 [8 warps][D/4]
    static __host__ __device__ uint32_t bar(int M) { return red(M) + 8 * (D / 4) * 4; }       // u64
    static __host__ __device__ uint32_t tslot(int M) { return bar(M) + 8; }                   // u32
    static __host__ __device__ uint32_t bytes(int M) { return tslot(M) + 16 + 1024; }
};

// Instruction descriptor (kind::f16, bf16 inputs, fp32 accumulator) with the
// major-ness of both operands: bit 15 transposes A (MN-major), bit 16 B.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_ab(int M, int N, bool a_mn_major, bool b_mn_major)
{
    return idesc_bf16_f32(M, N, b_mn_major) | ((a_mn_major ? 1u : 0u) << 15);
}

// dst[0..3] += v (fp32 reduction in L2, no return value).
__device__ __forceinline__ void red_add_v4(float *dst, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// One d-vector (bf16) in fp32 rotated by R(i, j): table[pos * D/4 + k] holds
// (cos, sin) of pos * theta_k.
template <int D>
__device__ __forceinline__ void load_rotated_f32(const __nv_bfloat16 *__restrict__ src, const float2 *table, int i,
                                                 int j, float (&x)[D])
{
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
            const float2 ry = table[i * (D / 4) + k], rx = table[j * (D / 4) + k];
            const float a0 = x[2 * k], a1 = x[2 * k + 1];
            x[2 * k] = a0 * ry.x - a1 * ry.y;
            x[2 * k + 1] = a0 * ry.y + a1 * ry.x;
            const float b0 = x[D / 2 + 2 * k], b1 = x[D / 2 + 2 * k + 1];
            x[D / 2 + 2 * k] = b0 * rx.x - b1 * rx.y;
            x[D / 2 + 2 * k + 1] = b0 * rx.y + b1 * rx.x;
        }
    }
}

// The gradient g = dL/d(R x) of a rotated vector x~ = R(i, j) x: adds the
// theta gradient of its pairs to dth[k] and turns g back by R(-i, -j) in
// place (the gradient with respect to x).
template <int D>
__device__ __forceinline__ void unrotate_grad(float (&g)[D], const float (&xr)[D], const float2 *table, int i, int j,
                                              float (&dth)[D / 4])
{
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
        const int a0 = 2 * k, a1 = 2 * k + 1, b0 = D / 2 + 2 * k, b1 = D / 2 + 2 * k + 1;
        dth[k] += (float)i * (g[a1] * xr[a0] - g[a0] * xr[a1]) + (float)j * (g[b1] * xr[b0] - g[b0] * xr[b1]);
        const float2 ry = table[i * (D / 4) + k], rx = table[j * (D / 4) + k];
        // R(-a) (g0, g1) = (g0 cos a + g1 sin a, -g0 sin a + g1 cos a)
        const float y0 = g[a0] * ry.x + g[a1] * ry.y, y1 = g[a1] * ry.x - g[a0] * ry.y;
        g[a0] = y0;
        g[a1] = y1;
        const float x0 = g[b0] * rx.x + g[b1] * rx.y, x1 = g[b1] * rx.x - g[b0] * rx.y;
        g[b0] = x0;
        g[b1] = x1;
    }
}

template <int D>
__device__ __forceinline__ void store_bf16_row(__nv_bfloat16 *dst, const float (&x)[D])
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < D / 8; ++c)
        d4[c] = make_uint4(pack_bf16x2(x[8 * c + 0], x[8 * c + 1]), pack_bf16x2(x[8 * c + 2], x[8 * c + 3]),
                           pack_bf16x2(x[8 * c + 4], x[8 * c + 5]), pack_bf16x2(x[8 * c + 6], x[8 * c + 7]));
}

// Sum of dth[k] over the CTA's NW warps, added to dtheta[k] (one reduction
// per frequency and CTA).
template <int D, int NW>
__device__ __forceinline__ void cta_add_dtheta(float (&dth)[D / 4], float *red_smem, float *dtheta_h)
{
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
        float v = dth[k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0)
            red_smem[warp * (D / 4) + k] = v;
    }
    __syncthreads();
    if (t < D / 4) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            sum += red_smem[w * (D / 4) + t];
        atomicAdd(dtheta_h + t, sum);
    }
}

// One half (dims [HALF * D/2, HALF * D/2 + D/2)) of a d-vector (bf16), in
// fp32, rotated by R(i, j) when a table is given: the first half turns by
// i theta_k, the second by j theta_k, k < D/4.
template <int D>
__device__ __forceinline__ void load_half_rotated(const __nv_bfloat16 *__restrict__ src, const float2 *table,
                                                  int half, int i, int j, float (&x)[D / 2])
{
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src + half * (D / 2));
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
        const uint4 u = __ldg(s4 + c);
        x[8 * c + 0] = bf16lo(u.x); x[8 * c + 1] = bf16hi(u.x);
        x[8 * c + 2] = bf16lo(u.y); x[8 * c + 3] = bf16hi(u.y);
        x[8 * c + 4] = bf16lo(u.z); x[8 * c + 5] = bf16hi(u.z);
        x[8 * c + 6] = bf16lo(u.w); x[8 * c + 7] = bf16hi(u.w);
    }
    if (table) {
        const int pos = half ? j : i;
#pragma unroll
        for (int k = 0; k < D / 4; ++k) {
            const float2 r = table[pos * (D / 4) + k];
            const float a0 = x[2 * k], a1 = x[2 * k + 1];
            x[2 * k] = a0 * r.x - a1 * r.y;
            x[2 * k + 1] = a0 * r.y + a1 * r.x;
        }
    }
}

// The gradient g = dL/d(R x) of one half of a rotated vector x~ (the half's
// pairs all turn by pos theta_k, pos = i for the first half, j for the
// second): adds pos (g1 x~0 - g0 x~1) to dth[k] and turns g back by
// R(-pos theta_k) in place.
template <int D>
__device__ __forceinline__ void unrotate_half(float (&g)[D / 2], const float (&xr)[D / 2], const float2 *table, int pos,
                                              float (&dth)[D / 4])
{
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
        const int a0 = 2 * k, a1 = 2 * k + 1;
        dth[k] += (float)pos * (g[a1] * xr[a0] - g[a0] * xr[a1]);
        const float2 r = table[pos * (D / 4) + k];
        // R(-a) (g0, g1) = (g0 cos a + g1 sin a, -g0 sin a + g1 cos a)
        const float y0 = g[a0] * r.x + g[a1] * r.y, y1 = g[a1] * r.x - g[a0] * r.y;
        g[a0] = y0;
        g[a1] = y1;
    }
}

template <int N>
__device__ __forceinline__ void store_bf16_vec(__nv_bfloat16 *dst, const float (&x)[N])
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < N / 8; ++c)
        d4[c] = make_uint4(pack_bf16x2(x[8 * c + 0], x[8 * c + 1]), pack_bf16x2(x[8 * c + 2], x[8 * c + 3]),
                           pack_bf16x2(x[8 * c + 4], x[8 * c + 5]), pack_bf16x2(x[8 * c + 6], x[8 * c + 7]));
}

// N consecutive fp32 TMEM columns of this thread's lane (16 or 32).
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, float (&v)[N])
{
    static_assert(N == 16 || N == 32, "16 or 32 columns");
    if constexpr (N == 16)
        tmem_ld16(taddr, v);
    else
        tmem_ld32(taddr, v);
}

constexpr int kBwdThreads = 256;

// 256 threads: thread (half, t) with t = tid % 128 owns key row t (and query
// row t of the current query tile); the two halves split the gathers (K~, w
// | V; Q~, u | dO, D, lse), the query columns of the P / dS pass, and the two
// halves of the head dim when gradients leave (the RoPE pairs of a half turn
// by one coordinate, i or j).  Warps w and w + 4 share TMEM lane quarter
// w % 4 and read different columns of it.
template <int D, int R>
__global__ void __launch_bounds__(kBwdThreads)
    winattn_bwd_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                          const __nv_bfloat16 *__restrict__ v, const float *__restrict__ theta,
                          const __nv_bfloat16 *__restrict__ bias, const __nv_bfloat16 *__restrict__ o,
                          const __nv_bfloat16 *__restrict__ dout, const float *__restrict__ lse,
                          __nv_bfloat16 *__restrict__ dq, __nv_bfloat16 *__restrict__ dk,
                          __nv_bfloat16 *__restrict__ dv, float *__restrict__ dtheta, float *__restrict__ dbias,
                          float *__restrict__ dq_acc, const Geometry g, const float scale)
{
    using L = BwdLayout<D, R>;
    constexpr int DH = D / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    float2 *table = reinterpret_cast<float2 *>(base + L::TB);
    float *q_lse = reinterpret_cast<float *>(base + L::QI);
    float *q_dd = q_lse + 128;
    uint32_t *q_code = reinterpret_cast<uint32_t *>(q_dd + 128);
    float *red_smem = reinterpret_cast<float *>(base + L::red(g.M));
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + L::bar(g.M));
    uint32_t *tslot = reinterpret_cast<uint32_t *>(base + L::tslot(g.M));

    const int tid = threadIdx.x, warp = tid >> 5;
    const int t = tid & 127, half = tid >> 7;
    // a single query tile per window: the gradient accumulators reuse the
    // S^T / dP^T columns (256 columns, two CTAs per SM); otherwise dV and dK~
    // live past column 256
    const bool single = g.n_tiles == 1;
    const uint32_t ncols = single ? 256u : 512u;
    constexpr uint32_t cST = 0, cDP = 128;
    const uint32_t cDV = single ? 0u : 256u, cDK = cDV + D, cDQ = single ? (uint32_t)(2 * D + R) : 0u;

    if (warp == 0) {
        tmem_alloc(tslot, ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    const Item it = decode_item(g, blockIdx.x);
    const int kt = it.tile;
    if (theta) {
        for (int idx = tid; idx < g.M * (D / 4); idx += kBwdThreads) {
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
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float2 *tab = theta ? table : nullptr;
    float dth[D / 4];
#pragma unroll
    for (int e = 0; e < D / 4; ++e)
        dth[e] = 0.f;

    // ---- key row t: K~ (rotated, bf16) and w | V; its mask code
    const RowRef kr = tile_row(g, it.pack, kt, t);
    const TokenRef ktk = kr.valid ? token_ref(g, kr.w, kr.p, it.h) : TokenRef{};
    const bool kreal = kr.valid && !ktk.pad;
    const uint32_t kcode = kreal ? (uint32_t)((kr.slot << 2) | ktk.label) : 0xFFFEu;
    if (half == 0) {
        if (kreal) {
            gather_rotate_store<D>(k + ktk.offset, tab, ktk.i, ktk.j, 1.f, base + L::KT, t);
            if constexpr (R > 0)
                copy_row<R>(bias + (((int64_t)it.h * 2 + 1) * g.N + kr.p) * R, base + L::KB, t);
        } else {
            zero_row<D>(base + L::KT, t);
            if constexpr (R > 0)
                zero_row<R>(base + L::KB, t);
        }
    } else {
        if (kreal)
            copy_row<D>(v + ktk.offset, base + L::VT, t);
        else
            zero_row<D>(base + L::VT, t);
    }

    constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t kIdescDV = idesc_bf16_f32(128, D, true);              // A K-major, B MN-major
    constexpr uint32_t kIdescDQ = idesc_bf16_f32_ab(128, D, true, true);     // A MN-major, B MN-major
    constexpr uint32_t kIdescDVr = idesc_bf16_f32(128, R > 0 ? R : 16, true);
    constexpr uint32_t kIdescDQr = idesc_bf16_f32_ab(128, R > 0 ? R : 16, true, true);
    const float c2 = kLog2e;  // Q~ carries d^-1/2: the scores are z itself
    uint32_t phase = 0;
    bool ok = true;

    for (int qt = 0; qt < g.n_tiles && ok; ++qt) {
        // ---- 1. query row t: Q~, u | dO, D = dO . O, lse, mask code
        const RowRef qr = tile_row(g, it.pack, qt, t);
        const TokenRef qtk = qr.valid ? token_ref(g, qr.w, qr.p, it.h) : TokenRef{};
        const bool qreal = qr.valid && !qtk.pad;
        if (half == 0) {
            if (qreal) {
                gather_rotate_store<D>(q + qtk.offset, tab, qtk.i, qtk.j, scale, base + L::QT, t);
                if constexpr (R > 0)
                    copy_row<R>(bias + (((int64_t)it.h * 2 + 0) * g.N + qr.p) * R, base + L::QB, t);
            } else {
                zero_row<D>(base + L::QT, t);
                if constexpr (R > 0)
                    zero_row<R>(base + L::QB, t);
            }
        } else if (qreal) {
            copy_row<D>(dout + qtk.offset, base + L::OT, t);
            const uint4 *o4 = reinterpret_cast<const uint4 *>(o + qtk.offset);
            const uint4 *g4 = reinterpret_cast<const uint4 *>(dout + qtk.offset);
            float dd = 0.f;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 a = __ldg(o4 + c), b = __ldg(g4 + c);
                dd += bf16lo(a.x) * bf16lo(b.x) + bf16hi(a.x) * bf16hi(b.x) + bf16lo(a.y) * bf16lo(b.y) +
                      bf16hi(a.y) * bf16hi(b.y) + bf16lo(a.z) * bf16lo(b.z) + bf16hi(a.z) * bf16hi(b.z) +
                      bf16lo(a.w) * bf16lo(b.w) + bf16hi(a.w) * bf16hi(b.w);
            }
            q_dd[t] = dd;
            q_lse[t] = __ldg(lse + qtk.offset / D) * kLog2e;
            q_code[t] = (uint32_t)((qr.slot << 2) | qtk.label);
        } else {
            zero_row<D>(base + L::OT, t);
            q_dd[t] = 0.f;
            q_lse[t] = 0.f;
            q_code[t] = 0xFFFFu;
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- 2. S^T = K~ Q~^T, dP^T = V dO^T
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t a = smem_desc(sbase + L::KT + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                const uint64_t b = smem_desc(sbase + L::QT + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                umma_bf16_ss(tmem + cST, a, b, kIdescS, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < R / 16; ++ks) {
                const uint64_t a = smem_desc(sbase + L::KB + ks * 32, 16, 16 * R, swizzle_code(2 * R));
                const uint64_t b = smem_desc(sbase + L::QB + ks * 32, 16, 16 * R, swizzle_code(2 * R));
                umma_bf16_ss(tmem + cST, a, b, kIdescS, 1);
            }
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t a = smem_desc(sbase + L::VT + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                const uint64_t b = smem_desc(sbase + L::OT + ks * 32, 16, 16 * D, swizzle_code(2 * D));
                umma_bf16_ss(tmem + cDP, a, b, kIdescS, ks > 0);
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

        // ---- 3. P^T and dS^T of key row t: this half's 64 queries, 32 at a time
#pragma unroll 1
        for (int c = 2 * half; c < 2 * half + 2; ++c) {
            float s[32], dp[32];
            tmem_ld32(tmem + lane_off + cST + c * 32, s);
            tmem_ld32(tmem + lane_off + cDP + c * 32, dp);
            uint32_t pk[16], dk2[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                float p2[2], d2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int col = 32 * c + e + u;
                    const bool allowed = q_code[col] == kcode;
                    const float p = allowed ? fast_exp2(fmaf(s[e + u], c2, -q_lse[col])) : 0.f;
                    p2[u] = p;
                    d2[u] = p * (dp[e + u] - q_dd[col]);
                }
                pk[e >> 1] = pack_bf16x2(p2[0], p2[1]);
                dk2[e >> 1] = pack_bf16x2(d2[0], d2[1]);
            }
            // columns [32 c, 32 c + 32): four 16-byte chunks of atom c / 2
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int chunk = (c & 1) * 4 + ch;
                const uint32_t off = (uint32_t)(c >> 1) * 16384u + swz_offset(t, chunk, 128);
                *reinterpret_cast<uint4 *>(base + L::PT + off) =
                    make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
                *reinterpret_cast<uint4 *>(base + L::DS + off) =
                    make_uint4(dk2[4 * ch], dk2[4 * ch + 1], dk2[4 * ch + 2], dk2[4 * ch + 3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- 4. dV += P^T dO, dK~ += dS^T Q~, dQ~ = dS K~
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                // A K-major over 16 queries: atom ks / 4, +32 bytes per step inside it
                const uint32_t aoff = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                const uint64_t ap = smem_desc(sbase + L::PT + aoff, 16, 1024, 2);
                const uint64_t ad = smem_desc(sbase + L::DS + aoff, 16, 1024, 2);
                const uint32_t acc = (qt > 0 || ks > 0) ? 1u : 0u;
                // B MN-major over 16 query rows of dO / Q~: +32 D bytes per step
                const uint64_t bo = smem_desc(sbase + L::OT + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D));
                const uint64_t bq = smem_desc(sbase + L::QT + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D));
                umma_bf16_ss(tmem + cDV, ap, bo, kIdescDV, acc);
                umma_bf16_ss(tmem + cDK, ad, bq, kIdescDV, acc);
                if constexpr (R > 0) {
                    const uint64_t bqb = smem_desc(sbase + L::QB + ks * 32 * R, 8192, 16 * R, swizzle_code(2 * R));
                    umma_bf16_ss(tmem + cDK + D, ad, bqb, kIdescDVr, acc);
                }
                // dS as the A operand (queries x keys): MN-major over the
                // dS^T tile, 16 key rows (2048 bytes) per step; the two
                // 64-query atoms are 16384 bytes apart
                const uint64_t at = smem_desc(sbase + L::DS + ks * 2048, 16384, 1024, 2);
                const uint64_t bk = smem_desc(sbase + L::KT + ks * 32 * D, 8192, 16 * D, swizzle_code(2 * D));
                umma_bf16_ss(tmem + cDQ, at, bk, kIdescDQ, ks > 0);
                if constexpr (R > 0) {
                    const uint64_t bkb = smem_desc(sbase + L::KB + ks * 32 * R, 8192, 16 * R, swizzle_code(2 * R));
                    umma_bf16_ss(tmem + cDQ + D, at, bkb, kIdescDQr, ks > 0);
                }
            }
            umma_commit(bar);
        }
        const bool g_done = mbar_wait(bar, phase);
        phase ^= 1;
        if (__syncthreads_or(!g_done)) {
            ok = false;
            break;
        }
        tc_fence_after_sync();

        // ---- 5. dQ~ of query row t (TMEM lane t): this half's head dims
        {
            float gq[DH];
            tmem_ldn<DH>(tmem + lane_off + cDQ + half * DH, gq);
            float gu[R > 0 ? R : 1];
            if constexpr (R == 16)
                tmem_ld16(tmem + lane_off + cDQ + D, gu);
            if constexpr (R == 32)
                tmem_ld32(tmem + lane_off + cDQ + D, gu);
            if (qreal) {
                if constexpr (R > 0) {
                    if (half == 0) {
                        float *du = dbias + (((int64_t)it.h * 2 + 0) * g.N + qr.p) * R;
#pragma unroll
                        for (int e = 0; e < R; e += 4)
                            red_add_v4(du + e, gu[e], gu[e + 1], gu[e + 2], gu[e + 3]);
                    }
                }
                if (single) {
#pragma unroll
                    for (int e = 0; e < DH; ++e)
                        gq[e] *= scale;
                    if (tab) {
                        float xr[DH];
                        load_half_rotated<D>(q + qtk.offset, tab, half, qtk.i, qtk.j, xr);
                        unrotate_half<D>(gq, xr, tab, half ? qtk.j : qtk.i, dth);
                    }
                    store_bf16_vec<DH>(dq + qtk.offset + half * DH, gq);
                } else {
                    float *acc = dq_acc + qtk.offset + half * DH;
#pragma unroll
                    for (int e = 0; e < DH; e += 4)
                        red_add_v4(acc + e, gq[e], gq[e + 1], gq[e + 2], gq[e + 3]);
                }
            }
        }
        // the tiles and TMEM columns are rewritten by the next query tile
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    }

    // ---- dV, dK of key row t: this half's head dims
    if (ok) {
        float gv[DH], gk[DH];
        tmem_ldn<DH>(tmem + lane_off + cDV + half * DH, gv);
        tmem_ldn<DH>(tmem + lane_off + cDK + half * DH, gk);
        float gw[R > 0 ? R : 1];
        if constexpr (R == 16)
            tmem_ld16(tmem + lane_off + cDK + D, gw);
        if constexpr (R == 32)
            tmem_ld32(tmem + lane_off + cDK + D, gw);
        if (kreal) {
            store_bf16_vec<DH>(dv + ktk.offset + half * DH, gv);
            if (tab) {
                float xr[DH];
                load_half_rotated<D>(k + ktk.offset, tab, half, ktk.i, ktk.j, xr);
                unrotate_half<D>(gk, xr, tab, half ? ktk.j : ktk.i, dth);
            }
            store_bf16_vec<DH>(dk + ktk.offset + half * DH, gk);
            if constexpr (R > 0) {
                if (half == 0) {
                    float *dw = dbias + (((int64_t)it.h * 2 + 1) * g.N + kr.p) * R;
#pragma unroll
                    for (int e = 0; e < R; e += 4)
                        red_add_v4(dw + e, gw[e], gw[e + 1], gw[e + 2], gw[e + 3]);
                }
            }
        }
        if (tab && dtheta)
            cta_add_dtheta<D, kBwdThreads / 32>(dth, red_smem, dtheta + it.h * (D / 4));
    } else if (tid == 0) {
        atomicOr(&g_status_word, 1u);
        // give an MMA that may still be in flight one more bounded chance to
        // land before its TMEM is released
        mbar_wait(bar, phase);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, ncols);
    }
}

// Windows of more than one query tile: dq from the summed dQ~ of every key
// tile (fp32 workspace, without d^-1/2), and the query side of the theta
// gradient.  Grid (token blocks, heads): every thread of a block has the
// same head.
template <int D>
__global__ void __launch_bounds__(128)
    winattn_bwd_finalize_kernel(const __nv_bfloat16 *__restrict__ q, const float *__restrict__ theta,
                                const float *__restrict__ dq_acc, __nv_bfloat16 *__restrict__ dq,
                                float *__restrict__ dtheta, const Geometry g, const float scale)
{
    __shared__ float red_smem[4 * (D / 4)];
    const int h = blockIdx.y;
    const int64_t tok = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t T = (int64_t)g.B * g.H * g.W;
    float dth[D / 4];
#pragma unroll
    for (int e = 0; e < D / 4; ++e)
        dth[e] = 0.f;
    if (tok < T) {
        const int64_t off = (tok * g.heads + h) * D;
        float gq[D];
#pragma unroll
        for (int e = 0; e < D; e += 4) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(dq_acc + off + e));
            gq[e] = a.x * scale;
            gq[e + 1] = a.y * scale;
            gq[e + 2] = a.z * scale;
            gq[e + 3] = a.w * scale;
        }
        if (theta) {
            // window-local (i, j) of the token: its position in the rolled grid
            const int x = (int)(tok % g.W), y = (int)((tok / g.W) % g.H);
            int yr = y - g.shift, xr = x - g.shift;
            if (yr < 0) yr += g.Hp;
            if (xr < 0) xr += g.Wp;
            const int i = yr % g.M, j = xr % g.M;
            float2 tab[2 * (D / 4)];  // (cos, sin) of i theta_k at [0, D/4), of j theta_k after
            float xq[D];
#pragma unroll
            for (int kk = 0; kk < D / 4; ++kk) {
                const float th = __ldg(theta + h * (D / 4) + kk);
                float sn, cs;
                sincosf((float)i * th, &sn, &cs);
                tab[kk] = make_float2(cs, sn);
                sincosf((float)j * th, &sn, &cs);
                tab[D / 4 + kk] = make_float2(cs, sn);
            }
            const uint4 *s4 = reinterpret_cast<const uint4 *>(q + off);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 u = __ldg(s4 + c);
                xq[8 * c + 0] = bf16lo(u.x); xq[8 * c + 1] = bf16hi(u.x);
                xq[8 * c + 2] = bf16lo(u.y); xq[8 * c + 3] = bf16hi(u.y);
                xq[8 * c + 4] = bf16lo(u.z); xq[8 * c + 5] = bf16hi(u.z);
                xq[8 * c + 6] = bf16lo(u.w); xq[8 * c + 7] = bf16hi(u.w);
            }
#pragma unroll
            for (int kk = 0; kk < D / 4; ++kk) {
                const int a0 = 2 * kk, a1 = a0 + 1, b0 = D / 2 + 2 * kk, b1 = b0 + 1;
                const float2 ry = tab[kk], rx = tab[D / 4 + kk];
                // x~ = R(i, j) x
                const float qa0 = xq[a0] * ry.x - xq[a1] * ry.y, qa1 = xq[a0] * ry.y + xq[a1] * ry.x;
                const float qb0 = xq[b0] * rx.x - xq[b1] * rx.y, qb1 = xq[b0] * rx.y + xq[b1] * rx.x;
                dth[kk] += (float)i * (gq[a1] * qa0 - gq[a0] * qa1) + (float)j * (gq[b1] * qb0 - gq[b0] * qb1);
                const float y0 = gq[a0] * ry.x + gq[a1] * ry.y, y1 = gq[a1] * ry.x - gq[a0] * ry.y;
                const float z0 = gq[b0] * rx.x + gq[b1] * rx.y, z1 = gq[b1] * rx.x - gq[b0] * rx.y;
                gq[a0] = y0;
                gq[a1] = y1;
                gq[b0] = z0;
                gq[b1] = z1;
            }
        }
        store_bf16_row<D>(dq + off, gq);
    }
    if (theta && dtheta)
        cta_add_dtheta<D, 4>(dth, red_smem, dtheta + h * (D / 4));
}

}  // namespace winattn
