// fp32 window-attention forward on the FP32 pipes (no tensor cores: the
// fp32 contract needs full single precision, which TF32 UMMA does not give).
//
// Same work decomposition as the tensor-core kernel: one CTA of 128 threads
// per 128-row query tile, thread t owns query row t.  Keys and values are
// staged 64 at a time in shared memory (keys already rotated); each thread
// runs an exact online softmax over its allowed keys with expf.
#pragma once
#include <cstdint>

#include "geometry.cuh"

namespace winattn {

constexpr int kSimtKeys = 64;

template <int D, int R>
struct SimtLayout {
    static constexpr uint32_t KS = 0;                              // keys    [64][D + R] fp32
    static constexpr uint32_t VS = KS + kSimtKeys * (D + R) * 4;   // values  [64][D]     fp32
    static constexpr uint32_t CS = VS + kSimtKeys * D * 4;         // codes   [64]        u16
    static constexpr uint32_t TB = CS + 2 * kSimtKeys;             // RoPE table [M][D/4] float2
    static __host__ __device__ uint32_t bytes(int M) { return TB + (uint32_t)(M * (D / 4) * 8) + 16; }
};

template <int D>
__device__ __forceinline__ void rotate_f32(float *x, const float2 *table, int i, int j)
{
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

template <int D, int R>
__global__ void __launch_bounds__(128)
    winattn_fwd_simt_kernel(const float *__restrict__ q, const float *__restrict__ k,
                            const float *__restrict__ v, const float *__restrict__ theta,
                            const float *__restrict__ bias, float *__restrict__ out, float *__restrict__ lse,
                            const Geometry g, const float scale)
{
    using L = SimtLayout<D, R>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    float *ks = reinterpret_cast<float *>(smem_raw + L::KS);
    float *vs = reinterpret_cast<float *>(smem_raw + L::VS);
    uint16_t *cs = reinterpret_cast<uint16_t *>(smem_raw + L::CS);
    float2 *table = reinterpret_cast<float2 *>(smem_raw + L::TB);
    const int t = threadIdx.x;
    const Item it = decode_item(g, blockIdx.x);

    if (theta) {
        for (int idx = t; idx < g.M * (D / 4); idx += blockDim.x) {
            const int c = idx / (D / 4), kk = idx - c * (D / 4);
            float sn, cn;
            sincosf((float)c * __ldg(theta + it.h * (D / 4) + kk), &sn, &cn);
            table[idx] = make_float2(cn, sn);
        }
    }
    __syncthreads();

    // query row t: rotated, content scaled by d^-1/2, factors u unscaled
    const RowRef qr = tile_row(g, it.pack, it.tile, t);
    float qv[D + R];
    int qcode = 0xFFFF;
    TokenRef qt{};
    if (qr.valid)
        qt = token_ref(g, qr.w, qr.p, it.h);
    const bool qreal = qr.valid && !qt.pad;  // a pad row of a padded grid has no output
    if (qreal) {
        qcode = (qr.slot << 2) | qt.label;
#pragma unroll
        for (int e = 0; e < D; ++e)
            qv[e] = __ldg(q + qt.offset + e);
        if (theta)
            rotate_f32<D>(qv, table, qt.i, qt.j);
#pragma unroll
        for (int e = 0; e < D; ++e)
            qv[e] *= scale;
#pragma unroll
        for (int e = 0; e < R; ++e)
            qv[D + e] = __ldg(bias + (((int64_t)it.h * 2 + 0) * g.N + qr.p) * R + e);
    } else {
#pragma unroll
        for (int e = 0; e < D + R; ++e)
            qv[e] = 0.f;
    }

    float m = -INFINITY, l = 0.f;
    float o[D];
#pragma unroll
    for (int e = 0; e < D; ++e)
        o[e] = 0.f;

    const int key_rows = g.U > 1 ? kTileRows : g.N;
    for (int k0 = 0; k0 < key_rows; k0 += kSimtKeys) {
        __syncthreads();
        if (t < kSimtKeys) {
            const int kk = k0 + t;
            uint16_t code = 0xFFFE;
            float *kr = ks + t * (D + R);
            float *vr = vs + t * D;
            if (kk < key_rows) {
                const RowRef rr = tile_row(g, it.pack, kk / kTileRows, kk % kTileRows);
                const TokenRef tk = rr.valid ? token_ref(g, rr.w, rr.p, it.h) : TokenRef{};
                if (rr.valid && !tk.pad) {
                    code = (uint16_t)((rr.slot << 2) | tk.label);
                    float x[D];
#pragma unroll
                    for (int e = 0; e < D; ++e)
                        x[e] = __ldg(k + tk.offset + e);
                    if (theta)
                        rotate_f32<D>(x, table, tk.i, tk.j);
#pragma unroll
                    for (int e = 0; e < D; ++e) {
                        kr[e] = x[e];
                        vr[e] = __ldg(v + tk.offset + e);
                    }
#pragma unroll
                    for (int e = 0; e < R; ++e)
                        kr[D + e] = __ldg(bias + (((int64_t)it.h * 2 + 1) * g.N + rr.p) * R + e);
                }
            }
            cs[t] = code;
        }
        __syncthreads();
        const int nk = min(kSimtKeys, key_rows - k0);
        for (int c = 0; c < nk; ++c) {
            if (cs[c] != qcode)
                continue;
            const float *kr = ks + c * (D + R);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < D + R; ++e)
                s = fmaf(qv[e], kr[e], s);
            const float m_new = fmaxf(m, s);
            const float corr = expf(m - m_new);
            const float p = expf(s - m_new);
            l = l * corr + p;
            const float *vr = vs + c * D;
#pragma unroll
            for (int e = 0; e < D; ++e)
                o[e] = fmaf(o[e], corr, p * vr[e]);
            m = m_new;
        }
    }
    if (qreal) {
        const float inv = 1.f / l;
        if (lse)
            lse[qt.offset / D] = m + logf(l);
#pragma unroll
        for (int e = 0; e < D; ++e)
            out[qt.offset + e] = o[e] * inv;
    }
}

}  // namespace winattn
