// Window geometry shared by the host planner and the kernels: how units
// (image b, window (wy, wx), head h) are packed into 128-row tiles and how a
// tile row maps to a token of the original B x H x W map.
//
// The cyclic shift is applied by index ("FLASHSWIN", section "어떻게 동작하나":
// shifted windows are recomputed per window after a cyclic move): rolled
// token (yr, xr) is original token ((yr + shift) mod H, (xr + shift) mod W),
// so no rolled copy of the map is ever made, and the write-back goes to the
// same original position (the inverse roll).
#pragma once
#include <cstdint>

namespace winattn {

constexpr int kTileRows = 128;  // rows of a query tile / key tile (UMMA M and N)

struct Geometry {
    int B, H, W, M, shift, heads, d, rank;
    int nWy, nWx;      // windows per image along rows / columns
    int N;             // tokens per window, M*M
    int U;             // windows packed into one tile (>= 1; > 1 only when N <= 64)
    int n_tiles;       // query tiles (and key tiles) per window when U == 1, else 1
    int64_t wph;       // windows per head, B * nWy * nWx
    int64_t packs;     // tiles per head along the window axis, ceil(wph / U)
    int64_t items;     // work items: heads * packs * n_tiles

    __host__ __device__ static Geometry make(int B, int H, int W, int M, int shift, int heads, int d, int rank)
    {
        Geometry g;
        g.B = B; g.H = H; g.W = W; g.M = M; g.shift = shift; g.heads = heads; g.d = d; g.rank = rank;
        g.nWy = H / M;
        g.nWx = W / M;
        g.N = M * M;
        g.U = g.N >= kTileRows ? 1 : kTileRows / g.N;
        g.n_tiles = g.U > 1 ? 1 : (g.N + kTileRows - 1) / kTileRows;
        g.wph = (int64_t)B * g.nWy * g.nWx;
        g.packs = (g.wph + g.U - 1) / g.U;
        g.items = (int64_t)heads * g.packs * g.n_tiles;
        return g;
    }
};

struct Item {
    int h;          // head
    int64_t pack;   // window index (U == 1) or pack of U windows (U > 1), within the head
    int tile;       // query tile within the window (0 when U > 1)
};

// Items are ordered head-major, then window, then query tile, so the query
// tiles of one window run side by side (its keys and values stay in L2).
__host__ __device__ inline Item decode_item(const Geometry &g, int64_t item)
{
    Item it;
    it.tile = (int)(item % g.n_tiles);
    const int64_t rest = item / g.n_tiles;
    it.pack = rest % g.packs;
    it.h = (int)(rest / g.packs);
    return it;
}

struct RowRef {
    bool valid;     // row holds a real token
    int slot;       // window slot inside a packed tile
    int64_t w;      // window index within the head
    int p;          // window-local token index, p = i*M + j
};

// Row t of tile `tile` of pack/window `pack`.
__host__ __device__ inline RowRef tile_row(const Geometry &g, int64_t pack, int tile, int t)
{
    RowRef r;
    if (g.U > 1) {
        r.slot = t / g.N;
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
    int64_t offset;  // element offset of the (token, head) d-vector in the map
    int i, j;        // window-local row / column
    int label;       // wrap label: 2*[rolled row in last `shift` rows] + [rolled col in last `shift` cols]
};

__host__ __device__ inline TokenRef token_ref(const Geometry &g, int64_t w, int p, int h)
{
    TokenRef t;
    const int64_t per_img = (int64_t)g.nWy * g.nWx;
    const int b = (int)(w / per_img);
    const int rem = (int)(w - (int64_t)b * per_img);
    const int wy = rem / g.nWx;
    const int wx = rem - wy * g.nWx;
    t.i = p / g.M;
    t.j = p - t.i * g.M;
    const int yr = wy * g.M + t.i;
    const int xr = wx * g.M + t.j;
    int y = yr + g.shift;
    if (y >= g.H) y -= g.H;
    int x = xr + g.shift;
    if (x >= g.W) x -= g.W;
    t.label = g.shift ? 2 * (yr >= g.H - g.shift) + (xr >= g.W - g.shift) : 0;
    t.offset = ((((int64_t)b * g.H + y) * g.W + x) * g.heads + h) * g.d;
    return t;
}

}  // namespace winattn
