// The two pieces around the attention on the "Rank-Factorized Implicit
// Neural Bias: Scaling Super-Resolution Transformer with FlashAttention" page:
//
//  - section 2.1 (RIB): the rank-r factors u, w of each window position come
//    from Fourier features of its 2D coordinate through a light MLP.  The
//    table depends only on the window-local position and the head, so it is
//    generated once per call (a prologue kernel, 128 positions per CTA) and
//    read by every window's attention from L2, instead of being recomputed by
//    every CTA that needs a tile of it;
//  - section 2.2 (CLA): a gate sigmoid(PW1x1(DW3x3(x))) multiplies the
//    attention output.  One persistent kernel: per 128-token tile the
//    depth-wise 3 x 3 convolution on the CUDA cores (fp32, zero padding),
//    rounded to bf16 into a K-major operand tile, the C x C point-wise
//    contraction on tcgen05 into TMEM, then bias, sigmoid and the product with
//    O in the epilogue.
//
// Feature order and coordinates (the page gives no sizes): c = 2 i / (M - 1)
// - 1 per axis (0 when M = 1), 8 octaves, features [sin 2^k pi c_y]_k,
// [cos 2^k pi c_y]_k, [sin 2^k pi c_x]_k, [cos 2^k pi c_x]_k; hidden width 64,
// tanh, no biases.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace winattn {

constexpr int kRibFeatures = 32, kRibHidden = 64;

// table [heads][2][M*M][R] bf16 from w1 [heads][2][32][64], w2 [heads][2][64][R]
// (fp32).  Grid (ceil(M*M / 128), heads * 2), 128 threads: one position each.
template <int R>
__global__ void __launch_bounds__(128)
    winattn_rib_features_kernel(const float *__restrict__ w1, const float *__restrict__ w2, int M,
                                __nv_bfloat16 *__restrict__ table)
{
    __shared__ float a[kRibFeatures * kRibHidden];
    __shared__ float b[kRibHidden * R];
    const int hs = blockIdx.y;  // head * 2 + side
    const float *a_src = w1 + (size_t)hs * kRibFeatures * kRibHidden;
    const float *b_src = w2 + (size_t)hs * kRibHidden * R;
    for (int i = threadIdx.x; i < kRibFeatures * kRibHidden; i += blockDim.x)
        a[i] = __ldg(a_src + i);
    for (int i = threadIdx.x; i < kRibHidden * R; i += blockDim.x)
        b[i] = __ldg(b_src + i);
    __syncthreads();
    const int N = M * M;
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= N)
        return;
    const int i = p / M, j = p - (p / M) * M;
    const float cy = M > 1 ? 2.f * (float)i / (float)(M - 1) - 1.f : 0.f;
    const float cx = M > 1 ? 2.f * (float)j / (float)(M - 1) - 1.f : 0.f;
    float f[kRibFeatures];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        // sin(2^k pi c) as sinpi(2^k c): the power of two scales exactly
        const float sy = ldexpf(cy, k), sx = ldexpf(cx, k);
        f[k] = sinpif(sy);
        f[8 + k] = cospif(sy);
        f[16 + k] = sinpif(sx);
        f[24 + k] = cospif(sx);
    }
    float out[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
        out[r] = 0.f;
#pragma unroll 4
    for (int c = 0; c < kRibHidden; ++c) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < kRibFeatures; ++e)
            acc = fmaf(f[e], a[e * kRibHidden + c], acc);
        const float hdn = tanhf(acc);
#pragma unroll
        for (int r = 0; r < R; ++r)
            out[r] = fmaf(hdn, b[c * R + r], out[r]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(table + ((size_t)hs * N + p) * R);
#pragma unroll
    for (int r = 0; r < R; r += 8)
        dst[r / 8] = make_uint4(pack_bf16x2(out[r], out[r + 1]), pack_bf16x2(out[r + 2], out[r + 3]),
                                pack_bf16x2(out[r + 4], out[r + 5]), pack_bf16x2(out[r + 6], out[r + 7]));
}

// Shared memory of the gate kernel for C channels: the point-wise weights as
// the B operand (C_out rows, K = C_in), the depth-wise output tile as the A
// operand (128 rows, K = C), both K-major in 16-channel atoms of 32-byte
// rows (32-byte swizzle), then the per-channel biases and the barrier.
struct GateLayout {
    static __host__ __device__ uint32_t b_bytes(int C) { return (uint32_t)C * C * 2; }
    static __host__ __device__ uint32_t a_off(int C) { return (b_bytes(C) + 1023) & ~1023u; }
    static __host__ __device__ uint32_t bias_off(int C) { return a_off(C) + 128u * C * 2; }
    static __host__ __device__ uint32_t bar_off(int C) { return bias_off(C) + (uint32_t)C * 4 * 11; }
    static __host__ __device__ uint32_t bytes(int C) { return bar_off(C) + 16 + 1024; }
};

// out = o * sigmoid(pw (dw3x3(x) + dw_b) + pw_b) per token and channel;
// x, o, out bf16 [B][H][W][C] (out may be o); dw fp32 [C][3][3], dw_b [C],
// pw fp32 [C_out][C_in], pw_b [C].  Persistent: grid <= the SM count, tile =
// 128 consecutive tokens of the row-major map.  512 threads: thread
// (group, t) handles token t of the tile and the 16-channel atoms
// a = group (mod 4), so that 16 warps hide the gather latency; warps w,
// w + 4, w + 8, w + 12 share TMEM lane quarter w % 4 and read their own
// atoms' columns of it.
constexpr int kGateThreads = 512;

__global__ void __launch_bounds__(kGateThreads, 1)
    winattn_cla_gate_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *o,
                            const float *__restrict__ dw, const float *__restrict__ dw_b,
                            const float *__restrict__ pw, const float *__restrict__ pw_b, int B, int H, int W, int C,
                            __nv_bfloat16 *out)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(base);
    // depth-wise weights [9 taps][C] (a tap's 16 channels of an atom are four
    // float4 loads, the same address for every lane of a warp), then dw_b, pw_b
    float *s_dw = reinterpret_cast<float *>(base + GateLayout::bias_off(C));
    float *s_dwb = s_dw + 9 * C, *s_pwb = s_dwb + C;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + GateLayout::bar_off(C));
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int t = tid & 127, group = tid >> 7;  // token row of the tile, atom group
    const uint32_t ncols = C <= 32 ? 32u : (C <= 64 ? 64u : (C <= 128 ? 128u : 256u));
    if (warp == 0) {
        tmem_alloc(tslot, ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    // point-wise weights -> bf16 B operand: row co (output channel), 16-channel
    // input atoms of C_out rows x 32 bytes
    const int atoms = C / 16;
    for (int idx = tid; idx < C * atoms; idx += kGateThreads) {
        const int co = idx / atoms, a = idx - co * atoms;
        const float *src = pw + (size_t)co * C + a * 16;
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            pk[e] = pack_bf16x2(__ldg(src + 2 * e), __ldg(src + 2 * e + 1));
        uint8_t *dst = base + (uint32_t)a * C * 32;
        *reinterpret_cast<uint4 *>(dst + swz_offset(co, 0, 32)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4 *>(dst + swz_offset(co, 1, 32)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    for (int idx = tid; idx < 9 * C; idx += kGateThreads) {
        const int ch = idx / 9, tap = idx - ch * 9;
        s_dw[tap * C + ch] = __ldg(dw + idx);
    }
    for (int idx = tid; idx < C; idx += kGateThreads) {
        s_dwb[idx] = __ldg(dw_b + idx);
        s_pwb[idx] = __ldg(pw_b + idx);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t aoff = GateLayout::a_off(C);
    const uint32_t idesc = idesc_bf16_f32(128, C, false);
    const int64_t T = (int64_t)B * H * W;
    const int64_t tiles = (T + 127) / 128;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        // ---- depth-wise 3 x 3 of token `tok`, all channels, into A row t
        const int64_t tok = tile * 128 + t;
        const bool real = tok < T;
        int b = 0, r = 0, c = 0;
        if (real) {
            c = (int)(tok % W);
            r = (int)((tok / W) % H);
            b = (int)(tok / ((int64_t)W * H));
        }
        for (int a = group; a < atoms; a += 4) {
            float acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                acc[e] = s_dwb[a * 16 + e];
            if (real) {
#pragma unroll
                for (int dy = -1; dy <= 1; ++dy)
#pragma unroll
                    for (int dx = -1; dx <= 1; ++dx) {
                        const int rr = r + dy, cc = c + dx;
                        if (rr < 0 || rr >= H || cc < 0 || cc >= W)
                            continue;
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            x + (((int64_t)b * H + rr) * W + cc) * C + a * 16);
                        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
                        const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                        const int tap = (dy + 1) * 3 + (dx + 1);
                        const float4 *wt = reinterpret_cast<const float4 *>(s_dw + tap * C + a * 16);
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const float4 wq = wt[e4];
                            acc[4 * e4 + 0] = fmaf(wq.x, bf16lo(wv[2 * e4]), acc[4 * e4 + 0]);
                            acc[4 * e4 + 1] = fmaf(wq.y, bf16hi(wv[2 * e4]), acc[4 * e4 + 1]);
                            acc[4 * e4 + 2] = fmaf(wq.z, bf16lo(wv[2 * e4 + 1]), acc[4 * e4 + 2]);
                            acc[4 * e4 + 3] = fmaf(wq.w, bf16hi(wv[2 * e4 + 1]), acc[4 * e4 + 3]);
                        }
                    }
            }
            uint8_t *dst = base + aoff + (uint32_t)a * 128 * 32;
            *reinterpret_cast<uint4 *>(dst + swz_offset(t, 0, 32)) =
                make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
            *reinterpret_cast<uint4 *>(dst + swz_offset(t, 1, 32)) =
                make_uint4(pack_bf16x2(acc[8], acc[9]), pack_bf16x2(acc[10], acc[11]), pack_bf16x2(acc[12], acc[13]),
                           pack_bf16x2(acc[14], acc[15]));
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        // ---- point-wise: G = A PW^T over 16-channel atoms
        if (tid == 0) {
            tc_fence_after_sync();
            for (int a = 0; a < atoms; ++a) {
                const uint64_t ad = smem_desc(sbase + aoff + (uint32_t)a * 128 * 32, 16, 256, swizzle_code(32));
                const uint64_t bd = smem_desc(sbase + (uint32_t)a * C * 32, 16, 256, swizzle_code(32));
                umma_bf16_ss(tmem, ad, bd, idesc, a > 0);
            }
            umma_commit(bar);
        }
        const bool done = mbar_wait(bar, phase);
        phase ^= 1;
        if (__syncthreads_or(!done)) {
            ok = false;
            break;
        }
        tc_fence_after_sync();
        // ---- epilogue: out = o * sigmoid(G + pw_b), 16 channels at a time
        // (every lane of a warp runs the same atoms: the TMEM load is collective)
        for (int a = group; a < atoms; a += 4) {
            float gv[16];
            tmem_ld16(trow + a * 16, gv);  // every lane: the load is warp-collective
            if (real) {
                const uint4 *op = reinterpret_cast<const uint4 *>(o + tok * C + a * 16);
                const uint4 u0 = op[0], u1 = op[1];
                const uint32_t ov[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                uint32_t pk[8];
                const float4 *bq = reinterpret_cast<const float4 *>(s_pwb + a * 16);
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 bb = bq[e4];
                    const float g0 = 1.f / (1.f + __expf(-(gv[4 * e4] + bb.x)));
                    const float g1 = 1.f / (1.f + __expf(-(gv[4 * e4 + 1] + bb.y)));
                    const float g2 = 1.f / (1.f + __expf(-(gv[4 * e4 + 2] + bb.z)));
                    const float g3 = 1.f / (1.f + __expf(-(gv[4 * e4 + 3] + bb.w)));
                    pk[2 * e4] = pack_bf16x2(bf16lo(ov[2 * e4]) * g0, bf16hi(ov[2 * e4]) * g1);
                    pk[2 * e4 + 1] = pack_bf16x2(bf16lo(ov[2 * e4 + 1]) * g2, bf16hi(ov[2 * e4 + 1]) * g3);
                }
                uint4 *dp = reinterpret_cast<uint4 *>(out + tok * C + a * 16);
                dp[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dp[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        // the A tile and the TMEM columns are rewritten by the next tile
        tc_fence_before_sync();
        __syncthreads();
    }
    if (!ok && tid == 0) {
        atomicOr(&g_status_word, 1u);
        mbar_wait(bar, phase);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, ncols);
    }
}

}  // namespace winattn
