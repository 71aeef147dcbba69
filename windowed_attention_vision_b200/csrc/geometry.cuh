// Window geometry shared by the host planner and the kernels: how units
// (image b, window (wy, wx), head h) are packed into 128-row tiles and how a
// tile row maps to a token of the original B x H x W map.
//
// The cyclic shift is applied by index ("FLASHSWIN", section "어떻게 동작하나":
// shifted windows are recomputed per window after a cyclic move): rolled
// token (yr, xr) is original token ((yr + shift) mod H, (xr + shift) mod W),
// so no rolled copy of the map is ever made, and the write-back goes to the
// same original position (the inverse roll).
//
// A map whose sides are not multiples of M is padded at the bottom and right
// to Hp x Wp (the next multiples of M), and the padded grid is rolled and cut
// into windows (Swin pads before its roll); pad positions hold no token: they
// are masked as keys and never written.  Nothing is copied: a pad position is
// only a flag of the index math.
//
// Indices are 32-bit (the host rejects problems whose window or item counts
// reach 2^31); divisions by the problem's runtime sizes use precomputed
// multiply-shift reciprocals.
#pragma once
#include <cstdint>

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

namespace winattn {

#if defined(WINATTN_DEBUG) && defined(__CUDA_ARCH__)
// Debug builds (-DWINATTN_DEBUG) check every index formed here and every TMA
// box origin against the map; a violation sets kStatusBounds in the device
// status word (read by winattn_last_device_status) and the access is clamped
// into the map instead of trapping.
extern __device__ unsigned int g_status_word;
constexpr unsigned int kStatusBounds = 2u;
__device__ __forceinline__ bool debug_in_range(int64_t v, int64_t lo, int64_t hi)
{
    if (v >= lo && v < hi)
        return true;
    atomicOr(&g_status_word, kStatusBounds);
    return false;
}
#endif

constexpr int kTileRows = 128;  // rows of a query tile / key tile (UMMA M and N)

// Division by a fixed divisor d >= 1 for dividends n < 2^31: with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1, n / d equals
// (umulhi(n, m) + n) >> l (Granlund and Montgomery, "Division by invariant
// integers using multiplication", 1994).
struct FastDiv {
    uint32_t d = 1, mul = 1, shift = 0;

    __host__ __device__ FastDiv() {}
    __host__ __device__ explicit FastDiv(uint32_t divisor) : d(divisor)
    {
        shift = 0;
        while ((1ull << shift) < d)
            ++shift;
        mul = (uint32_t)((((1ull << 32) * ((1ull << shift) - d)) / d) + 1);
    }
    __host__ __device__ uint32_t div(uint32_t n) const
    {
#ifdef __CUDA_ARCH__
        const uint32_t hi = __umulhi(n, mul);
#else
        const uint32_t hi = (uint32_t)(((uint64_t)n * mul) >> 32);
#endif
        return (hi + n) >> shift;
    }
};

struct Geometry {
    int B, H, W, M, shift, heads, d, rank;
    int Hp, Wp;        // H, W rounded up to multiples of M (the padded grid)
    bool padded;       // Hp != H or Wp != W
    int nWy, nWx;      // windows per image along rows / columns
    int N;             // tokens per window, M*M
    int U;             // windows packed into one tile (>= 1; > 1 only when N <= 64)
    int n_tiles;       // query tiles (and key tiles) per window when U == 1, else 1
    int64_t wph;       // windows per head, B * nWy * nWx
    int64_t packs;     // tiles per head along the window axis, ceil(wph / U)
    int64_t items;     // work items: heads * packs * n_tiles
    FastDiv div_N, div_M, div_nWx, div_img, div_heads, div_tiles, div_packs;

    __host__ __device__ static Geometry make(int B, int H, int W, int M, int shift, int heads, int d, int rank)
    {
        Geometry g;
        g.B = B; g.H = H; g.W = W; g.M = M; g.shift = shift; g.heads = heads; g.d = d; g.rank = rank;
        g.nWy = (H + M - 1) / M;
        g.nWx = (W + M - 1) / M;
        g.Hp = g.nWy * M;
        g.Wp = g.nWx * M;
        g.padded = g.Hp != H || g.Wp != W;
        g.N = M * M;
        g.U = g.N >= kTileRows ? 1 : kTileRows / g.N;
        g.n_tiles = g.U > 1 ? 1 : (g.N + kTileRows - 1) / kTileRows;
        g.wph = (int64_t)B * g.nWy * g.nWx;
        g.packs = (g.wph + g.U - 1) / g.U;
        g.items = (int64_t)heads * g.packs * g.n_tiles;
        g.div_N = FastDiv((uint32_t)g.N);
        g.div_M = FastDiv((uint32_t)M);
        g.div_nWx = FastDiv((uint32_t)g.nWx);
        g.div_img = FastDiv((uint32_t)(g.nWy * g.nWx));
        g.div_heads = FastDiv((uint32_t)heads);
        g.div_tiles = FastDiv((uint32_t)g.n_tiles);
        g.div_packs = FastDiv((uint32_t)(g.packs < 0x7FFFFFFF ? g.packs : 1));
        return g;
    }
};

struct Item {
    int h;          // head
    int pack;       // window index (U == 1) or pack of U windows (U > 1), within the head
    int tile;       // query tile within the window (0 when U > 1)
};

// Head-major order (window, then query tile, innermost): used by the generic
// kernel, where the query tiles of one window run side by side.
__host__ __device__ inline Item decode_item(const Geometry &g, int item)
{
    Item it;
    const uint32_t rest = g.div_tiles.div((uint32_t)item);
    it.tile = item - (int)rest * g.n_tiles;
    const uint32_t hq = g.div_packs.div(rest);
    it.pack = (int)(rest - hq * (uint32_t)g.packs);
    it.h = (int)hq;
    return it;
}

// Pack-major, head-minor order (one tile per item): used by the small-window
// kernel, so the heads of a token - which share its DRAM lines - are read by
// neighbouring CTAs at the same time.
__host__ __device__ inline Item decode_item_head_minor(const Geometry &g, int item)
{
    Item it;
    const uint32_t pack = g.div_heads.div((uint32_t)item);
    it.pack = (int)pack;
    it.h = item - (int)pack * g.heads;
    it.tile = 0;
    return it;
}

struct RowRef {
    bool valid;     // row holds a real token
    int slot;       // window slot inside a packed tile
    int w;          // window index within the head
    int p;          // window-local token index, p = i*M + j
};

// Row t of tile `tile` of pack/window `pack`.
__host__ __device__ inline RowRef tile_row(const Geometry &g, int pack, int tile, int t)
{
    RowRef r;
    if (g.U > 1) {
        r.slot = (int)g.div_N.div((uint32_t)t);
        r.p = t - r.slot * g.N;
        r.w = pack * g.U + r.slot;
        r.valid = r.slot < g.U && r.w < g.wph;
    } else {
        r.slot = 0;
        r.p = tile * kTileRows + t;
        r.w = pack;
        r.valid = r.p < g.N;
    }
    return r;
}

struct TokenRef {
    int64_t offset;  // element offset of the (token, head) d-vector in the map (0 for a pad)
    int i, j;        // window-local row / column
    int label;       // wrap label: 2*[rolled row in last `shift` rows] + [rolled col in last `shift` cols]
    bool pad;        // a pad position of the padded grid: no token
};

__host__ __device__ inline TokenRef token_ref(const Geometry &g, int w, int p, int h)
{
    TokenRef t;
    const int b = (int)g.div_img.div((uint32_t)w);
    const int rem = w - b * g.nWy * g.nWx;
    const int wy = (int)g.div_nWx.div((uint32_t)rem);
    const int wx = rem - wy * g.nWx;
    t.i = (int)g.div_M.div((uint32_t)p);
    t.j = p - t.i * g.M;
    const int yr = wy * g.M + t.i;
    const int xr = wx * g.M + t.j;
    int y = yr + g.shift;
    if (y >= g.Hp) y -= g.Hp;
    int x = xr + g.shift;
    if (x >= g.Wp) x -= g.Wp;
    t.label = g.shift ? 2 * (yr >= g.Hp - g.shift) + (xr >= g.Wp - g.shift) : 0;
    t.pad = y >= g.H || x >= g.W;
    t.offset = t.pad ? 0 : ((((int64_t)b * g.H + y) * g.W + x) * g.heads + h) * g.d;
#if defined(WINATTN_DEBUG) && defined(__CUDA_ARCH__)
    // the (b, y, x, h) the index math formed lies in the (padded) map, the
    // window-local (i, j) in the window
    if (!debug_in_range(b, 0, g.B) || !debug_in_range(y, 0, g.Hp) || !debug_in_range(x, 0, g.Wp) ||
        !debug_in_range(h, 0, g.heads) || !debug_in_range(t.i, 0, g.M) || !debug_in_range(t.j, 0, g.M) ||
        !debug_in_range(t.offset, 0, (int64_t)g.B * g.H * g.W * g.heads * g.d)) {
        t.offset = 0;
        t.pad = true;
    }
#endif
    return t;
}

// Whether window w lies in the last window row or column of a shifted map
// (the only windows whose tokens carry different wrap labels).
__host__ __device__ inline bool window_wrapped(const Geometry &g, int w)
{
    if (g.shift == 0)
        return false;
    const int b = (int)g.div_img.div((uint32_t)w);
    const int rem = w - b * g.nWy * g.nWx;
    const int wy = (int)g.div_nWx.div((uint32_t)rem);
    const int wx = rem - wy * g.nWx;
    return wy == g.nWy - 1 || wx == g.nWx - 1;
}

}  // namespace winattn
