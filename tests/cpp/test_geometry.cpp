// Host-side checks of the kernels' index math (compiled with g++, no GPU):
// multiply-shift division, item decoding, tile rows and token addressing
// against plain integer arithmetic.
#include <cstdio>
#include <cstdlib>
#include <random>

#include "../../windowed_attention_vision_b200/csrc/geometry.cuh"

using namespace winattn;

static int failures = 0;
#define CHECK(cond, ...)                          \
    do {                                          \
        if (!(cond)) {                            \
            if (failures < 20) {                  \
                std::printf("FAIL %s:%d: ", __FILE__, __LINE__); \
                std::printf(__VA_ARGS__);         \
                std::printf("\n");                \
            }                                     \
            ++failures;                           \
        }                                         \
    } while (0)

static void check_fastdiv()
{
    std::mt19937_64 rng(1);
    for (uint32_t d = 1; d <= 70000; d += (d < 3000 ? 1 : 97)) {
        FastDiv f(d);
        for (uint32_t n = 0; n < 4096; ++n)
            CHECK(f.div(n) == n / d, "%u / %u", n, d);
        for (int r = 0; r < 200; ++r) {
            const uint32_t n = (uint32_t)(rng() & 0x7FFFFFFFu);
            CHECK(f.div(n) == n / d, "%u / %u", n, d);
        }
        for (uint32_t k = 1; k < 64; ++k) {  // around multiples of d
            const uint64_t m = (uint64_t)d * (0x7FFFFFFFu / d / k);
            for (int e = -1; e <= 1; ++e) {
                const int64_t n = (int64_t)m + e;
                if (n >= 0 && n < 0x80000000ll)
                    CHECK(f.div((uint32_t)n) == (uint32_t)n / d, "%lld / %u", (long long)n, d);
            }
        }
        const uint32_t top = 0x7FFFFFFFu;
        CHECK(f.div(top) == top / d, "top / %u", d);
    }
}

static void check_problem(int B, int H, int W, int M, int s, int heads, int d)
{
    const Geometry g = Geometry::make(B, H, W, M, s, heads, d, 0);
    // the grid is padded to multiples of M; pad positions hold no token
    const int nWy = (H + M - 1) / M, nWx = (W + M - 1) / M, N = M * M;
    const int Hp = nWy * M, Wp = nWx * M;
    CHECK(g.Hp == Hp && g.Wp == Wp && g.padded == (Hp != H || Wp != W), "padded grid");
    const int U = N >= 128 ? 1 : 128 / N;
    CHECK(g.U == U, "U");
    // every (pack, tile, row) maps to the token plain arithmetic gives
    for (int pack = 0; pack < g.packs; ++pack)
        for (int tile = 0; tile < g.n_tiles; ++tile)
            for (int t = 0; t < 128; ++t) {
                const RowRef r = tile_row(g, pack, tile, t);
                int slot = U > 1 ? t / N : 0;
                int p = U > 1 ? t % N : tile * 128 + t;
                int w = U > 1 ? pack * U + slot : pack;
                bool valid = U > 1 ? (slot < U && w < (long long)B * nWy * nWx) : p < N;
                CHECK(r.valid == valid, "valid");
                if (!valid)
                    continue;
                CHECK(r.slot == slot && r.p == p && r.w == w, "row mapping");
                for (int h = 0; h < heads; h += (heads > 1 ? heads - 1 : 1)) {
                    const TokenRef tk = token_ref(g, w, p, h);
                    const int b = w / (nWy * nWx), wy = (w % (nWy * nWx)) / nWx, wx = w % nWx;
                    const int i = p / M, j = p % M;
                    const int y = (wy * M + i + s) % Hp, x = (wx * M + j + s) % Wp;
                    const bool pad = y >= H || x >= W;
                    const long long off = pad ? 0 : ((((long long)b * H + y) * W + x) * heads + h) * d;
                    const int label = s ? 2 * (wy * M + i >= Hp - s) + (wx * M + j >= Wp - s) : 0;
                    CHECK(tk.pad == pad && tk.offset == off && tk.i == i && tk.j == j && tk.label == label,
                          "token_ref");
                    CHECK(window_wrapped(g, w) == (s > 0 && (wy == nWy - 1 || wx == nWx - 1)), "wrapped");
                }
            }
    for (int item = 0; item < g.items; ++item) {
        const Item a = decode_item(g, item);
        CHECK(a.tile == item % g.n_tiles && a.pack == (item / g.n_tiles) % g.packs &&
                  a.h == item / g.n_tiles / g.packs, "decode_item");
        if (g.n_tiles == 1) {
            const Item b = decode_item_head_minor(g, item);
            CHECK(b.pack == item / heads && b.h == item % heads && b.tile == 0, "decode_item_head_minor");
        }
    }
}

int main()
{
    check_fastdiv();
    check_problem(2, 56, 56, 8, 4, 3, 32);
    check_problem(1, 24, 8, 8, 3, 1, 32);
    check_problem(2, 14, 21, 7, 3, 2, 32);
    check_problem(1, 12, 8, 4, 2, 3, 32);
    check_problem(1, 9, 6, 3, 1, 2, 64);
    check_problem(2, 5, 7, 1, 0, 2, 32);
    check_problem(1, 20, 20, 10, 5, 2, 32);
    check_problem(1, 24, 24, 12, 6, 2, 32);
    check_problem(1, 64, 96, 32, 16, 3, 32);
    check_problem(1, 192, 96, 96, 48, 2, 64);
    // padded grids
    check_problem(2, 56, 56, 32, 16, 3, 32);
    check_problem(1, 56, 56, 16, 8, 2, 32);
    check_problem(2, 10, 13, 4, 2, 2, 32);
    check_problem(1, 5, 7, 3, 1, 1, 64);
    if (failures) {
        std::printf("%d failures\n", failures);
        return 1;
    }
    std::printf("OK\n");
    return 0;
}
