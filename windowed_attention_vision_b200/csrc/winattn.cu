// C ABI of the fused window-attention forward (declared in include/winattn.h):
// argument checks, launch planning, kernel dispatch, the host-buffer variant
// and the per-device status word of the bounded waits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/winattn.h"
#include "bwd_tc.cuh"
#include "fwd_large.cuh"
#include "fwd_pipe.cuh"
#include "fwd_pipe16.cuh"
#include "fwd_simt.cuh"
#include "fwd_small.cuh"
#include "fwd_tc.cuh"
#include "geometry.cuh"
#include "rib_cla.cuh"

namespace winattn {

namespace {

constexpr int kMaxM = 256;      // RoPE table and window index limits
constexpr int kThreads = 128;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int check_sizes(int B, int H, int W, int M, int shift, int heads, int d, int rank, int dtype)
{
    if (dtype != WINATTN_BF16 && dtype != WINATTN_FP32)
        return WINATTN_ERR_DTYPE;
    if (B <= 0 || H <= 0 || W <= 0 || M <= 0 || heads <= 0 || M > kMaxM)
        return WINATTN_ERR_ARG;
    if (shift < 0 || shift >= M)
        return WINATTN_ERR_ARG;
    if (dtype == WINATTN_BF16 && d != 32 && d != 64)
        return WINATTN_ERR_ARG;
    if (dtype == WINATTN_FP32 && d != 16 && d != 32 && d != 64)
        return WINATTN_ERR_ARG;
    if (rank != 0 && rank != 16 && rank != 32)
        return WINATTN_ERR_RANK;
    const Geometry g = Geometry::make(B, H, W, M, shift, heads, d, rank);
    const double elems = (double)B * H * W * heads * d;
    if (elems > 9.0e18 || g.items > 0x7FFFFFFFLL || g.wph > 0x7FFFFFFFLL)
        return WINATTN_ERR_SIZE;
    return WINATTN_OK;
}

size_t map_bytes(int B, int H, int W, int heads, int d, int dtype)
{
    return (size_t)B * H * W * heads * d * (dtype == WINATTN_BF16 ? 2 : 4);
}

int smem_bytes_for(const Geometry &g, int dtype)
{
    if (dtype == WINATTN_BF16) {
        switch (g.d * 100 + g.rank) {
        case 3200: return (int)TcLayout<32, 0>::bytes(g.M);
        case 3216: return (int)TcLayout<32, 16>::bytes(g.M);
        case 3232: return (int)TcLayout<32, 32>::bytes(g.M);
        case 6400: return (int)TcLayout<64, 0>::bytes(g.M);
        case 6416: return (int)TcLayout<64, 16>::bytes(g.M);
        case 6432: return (int)TcLayout<64, 32>::bytes(g.M);
        }
    } else {
        switch (g.d * 100 + g.rank) {
        case 1600: return (int)SimtLayout<16, 0>::bytes(g.M);
        case 1616: return (int)SimtLayout<16, 16>::bytes(g.M);
        case 1632: return (int)SimtLayout<16, 32>::bytes(g.M);
        case 3200: return (int)SimtLayout<32, 0>::bytes(g.M);
        case 3216: return (int)SimtLayout<32, 16>::bytes(g.M);
        case 3232: return (int)SimtLayout<32, 32>::bytes(g.M);
        case 6400: return (int)SimtLayout<64, 0>::bytes(g.M);
        case 6416: return (int)SimtLayout<64, 16>::bytes(g.M);
        case 6432: return (int)SimtLayout<64, 32>::bytes(g.M);
        }
    }
    return -1;
}

constexpr int kAssumedSMs = 148;          // B200; used only by winattn_launch_info
constexpr uint32_t kMaxSmem = 227 * 1024;

enum KernelKind { kGeneric = 0, kSmall = 1, kLarge = 2, kSimt = 3, kPipe = 4, kPipe16 = 5, kKinds = 6 };

// Process-wide switches of the specialised kernels (winattn_set_kernel_enabled):
// a disabled kind's problems go to the generic kernel.  The generic and SIMT
// kernels cannot be disabled.
std::atomic<int> g_kernel_enabled[kKinds] = {1, 1, 1, 1, 1, 1};

bool kernel_enabled(KernelKind k) { return g_kernel_enabled[k].load(std::memory_order_relaxed) != 0; }

int current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return -1;
    return dev;
}

// cudaFuncAttributeMaxDynamicSharedMemorySize is a per-function, per-device
// setting: raised to the largest opt-in size once per (kernel, device) and
// never again (the launch itself passes the bytes it needs).
template <auto Kernel>
bool smem_attr_once()
{
    static std::atomic<uint64_t> done{0};
    const int dev = current_device();
    if (dev < 0)
        return false;
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit)
        return true;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
        return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
}

// Tensor maps of a launch depend only on the device, the buffers' addresses
// and the problem's sizes, so they are encoded once per such key and reused:
// a repeated key always denotes the same encoding, even after the caller has
// freed and reallocated a buffer at the same address.  A small table per
// process, replaced round-robin, guarded by a mutex (the lookup is a few
// hundred nanoseconds; encoding the 16 maps of an 8 x 8 window call costs
// several microseconds).
struct MapKey {
    int kind, dev, B, H, W, M, shift, heads, d, rank;
    const void *ptr[5];
    bool operator==(const MapKey &o) const { return std::memcmp(this, &o, sizeof *this) == 0; }
};

struct MapSet {
    alignas(64) CUtensorMap m[16];
};

constexpr int kMapCacheEntries = 64;

struct MapCache {
    std::mutex mu;
    MapKey key[kMapCacheEntries];
    MapSet val[kMapCacheEntries];
    bool used[kMapCacheEntries] = {};
    int next = 0;
};

MapCache &map_cache()
{
    static MapCache c;
    return c;
}

MapKey make_key(KernelKind kind, const Geometry &g, const void *a, const void *b, const void *c, const void *d,
                const void *e)
{
    MapKey k;
    std::memset(&k, 0, sizeof k);  // padding bytes take part in the comparison
    k.kind = kind;
    k.dev = current_device();
    k.B = g.B; k.H = g.H; k.W = g.W; k.M = g.M; k.shift = g.shift; k.heads = g.heads; k.d = g.d; k.rank = g.rank;
    k.ptr[0] = a; k.ptr[1] = b; k.ptr[2] = c; k.ptr[3] = d; k.ptr[4] = e;
    return k;
}

// The cached maps of `key`, or those `encode(MapSet *)` produces (then
// cached); false if encoding failed (nothing is cached then).
template <typename Encode>
bool cached_maps(const MapKey &key, MapSet *out, Encode encode)
{
    MapCache &c = map_cache();
    {
        std::lock_guard<std::mutex> lock(c.mu);
        for (int i = 0; i < kMapCacheEntries; ++i)
            if (c.used[i] && c.key[i] == key) {
                *out = c.val[i];
                return true;
            }
    }
    std::memset(out, 0, sizeof *out);
    if (!encode(out))
        return false;
    std::lock_guard<std::mutex> lock(c.mu);
    const int i = c.next;
    c.next = (c.next + 1) % kMapCacheEntries;
    c.key[i] = key;
    c.val[i] = *out;
    c.used[i] = true;
    return true;
}

uint32_t pipe_smem(const Geometry &g)
{
    return g.d == 32 ? PipeLayout<32>::bytes(g.heads) : PipeLayout<64>::bytes(g.heads);
}

uint32_t pipe16_smem(const Geometry &g)
{
    return g.d == 32 ? Pipe16Layout<32>::bytes(g.heads) : Pipe16Layout<64>::bytes(g.heads);
}

uint32_t small_smem(const Geometry &g)
{
    switch (g.d * 100 + g.rank) {
    case 3200: return SmallLayout<32, 0>::bytes(g.heads, g.M);
    case 3216: return SmallLayout<32, 16>::bytes(g.heads, g.M);
    case 3232: return SmallLayout<32, 32>::bytes(g.heads, g.M);
    case 6400: return SmallLayout<64, 0>::bytes(g.heads, g.M);
    case 6416: return SmallLayout<64, 16>::bytes(g.heads, g.M);
    case 6432: return SmallLayout<64, 32>::bytes(g.heads, g.M);
    }
    return ~0u;
}

// Which kernel serves a problem: windows of <= 128 tokens go to the
// persistent small-window kernel when its RoPE table and ring fit in shared
// memory; fp32 goes to the SIMT kernel; everything else to the generic one.
KernelKind choose_kernel(const Geometry &g, int dtype, bool want_lse = false)
{
    if (dtype == WINATTN_FP32)
        return kSimt;
    // the generic kernel resolves every token through the index math, pad
    // positions of a padded grid included; of the specialised kernels the
    // large-window one masks pad keys, and the 16 x 16 pipelined one serves
    // pads of half a window (whole key granules and store boxes)
    if (g.padded) {
        if (kernel_enabled(kPipe16) && pipe16_ok(g) && pipe16_smem(g) <= kMaxSmem)
            return kPipe16;
        return kernel_enabled(kLarge) && large_ok(g) ? kLarge : kGeneric;
    }
    if (kernel_enabled(kPipe) && pipe_ok(g) && (uint64_t)g.heads * g.M * (g.d / 4) * 8 <= kSmallTableMax &&
        pipe_smem(g) <= kMaxSmem)
        return kPipe;
    if (kernel_enabled(kPipe16) && pipe16_ok(g) && pipe16_smem(g) <= kMaxSmem)
        return kPipe16;
    // (the small-window kernel does not write the log-sum-exp)
    if (!want_lse && kernel_enabled(kSmall) && g.N <= kTileRows &&
        (uint64_t)g.heads * g.M * (g.d / 4) * 8 <= kSmallTableMax && small_smem(g) <= kMaxSmem)
        return kSmall;
    if (kernel_enabled(kLarge) && large_ok(g))
        return kLarge;
    return kGeneric;
}

int sm_count()
{
    static std::mutex mu;
    static int cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return kAssumedSMs;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = kAssumedSMs;
        cached[dev] = n;
    }
    return cached[dev];
}

// Compute capability check, cached per device.
int check_device()
{
    static std::mutex mu;
    static int cached[64];  // 0 unknown, 1 ok, 2 wrong arch
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return WINATTN_ERR_CUDA;
    if (dev < 0 || dev >= 64)
        return WINATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return WINATTN_ERR_CUDA;
        cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return cached[dev] == 1 ? WINATTN_OK : WINATTN_ERR_ARCH;
}

template <auto Kernel>
int launch(int smem, const Geometry &g, cudaStream_t stream, auto... args)
{
    if (!smem_attr_once<Kernel>())
        return WINATTN_ERR_CUDA;
    Kernel<<<(unsigned)g.items, kThreads, smem, stream>>>(args..., g, 1.0f / std::sqrt((float)g.d));
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

template <int D, int R>
int launch_tc(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
              float *lse, const Geometry &g, cudaStream_t stream)
{
    using T = __nv_bfloat16;
    constexpr auto kernel = winattn_fwd_tc_kernel<D, R, false>;
    if (!smem_attr_once<kernel>())
        return WINATTN_ERR_CUDA;
    kernel<<<(unsigned)g.items, kThreads, TcLayout<D, R>::bytes(g.M), stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), theta,
        static_cast<const T *>(bias), static_cast<T *>(out), lse, g, 1.0f / std::sqrt((float)g.d), nullptr, 0);
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 4-D view (channels, x, y, image) of a bf16 [B][H][W][heads*d] map with a
// (d, bw, bh, 1) box: one head's d-vector for a bw x bh rectangle of tokens,
// swizzled to match the d*2-byte rows of the UMMA operand tiles.
bool encode_window_map(CUtensorMap *m, const void *base, const Geometry &g, int bw, int bh)
{
    auto fn = tensor_map_encoder();
    if (!fn)
        return false;
    const cuuint64_t C = (cuuint64_t)g.heads * g.d;
    const cuuint64_t dims[4] = {C, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.B};
    const cuuint64_t strides[3] = {C * 2, C * 2 * g.W, C * 2 * g.W * g.H};
    const cuuint32_t box[4] = {(cuuint32_t)g.d, (cuuint32_t)bw, (cuuint32_t)bh, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          g.d == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The four box shapes of one operand (see WindowMaps).  All four are encoded
// whatever the shift: the pipelined kernel's epilogue stores half windows and
// quadrants of unshifted windows too.
bool encode_window_maps(WindowMaps *m, const void *base, const Geometry &g)
{
    if (!encode_window_map(&m->full, base, g, g.M, g.M))
        return false;
    const int hm = g.M / 2;
    return encode_window_map(&m->xhalf, base, g, hm, g.M) && encode_window_map(&m->yhalf, base, g, g.M, hm) &&
           encode_window_map(&m->quarter, base, g, hm, hm);
}

uint32_t large_layout_bytes(const Geometry &g)
{
    const bool b96 = large_tile_keys(g.M) == 96;
    switch (g.d * 100 + g.rank) {
    case 3200: return b96 ? LargeLayout<32, 0, 96>::BYTES : LargeLayout<32, 0, 128>::BYTES;
    case 3216: return b96 ? LargeLayout<32, 16, 96>::BYTES : LargeLayout<32, 16, 128>::BYTES;
    case 3232: return b96 ? LargeLayout<32, 32, 96>::BYTES : LargeLayout<32, 32, 128>::BYTES;
    case 6400: return b96 ? LargeLayout<64, 0, 96>::BYTES : LargeLayout<64, 0, 128>::BYTES;
    case 6416: return b96 ? LargeLayout<64, 16, 96>::BYTES : LargeLayout<64, 16, 128>::BYTES;
    case 6432: return b96 ? LargeLayout<64, 32, 96>::BYTES : LargeLayout<64, 32, 128>::BYTES;
    }
    return ~0u;
}

// Dynamic shared memory of a large-kernel launch: its layout, at least 116 KB
// so that one CTA (holding all of TMEM) is resident per SM.
uint32_t large_smem(const Geometry &g)
{
    const uint32_t need = large_layout_bytes(g);
    return need > 116u * 1024 ? need : 116u * 1024;
}

// 4-D K or V box map for the large-window kernel: (d, bw, rows, 1).
bool encode_kv_map(CUtensorMap *m, const void *base, const Geometry &g, int bw, int rows)
{
    auto fn = tensor_map_encoder();
    if (!fn)
        return false;
    const cuuint64_t C = (cuuint64_t)g.heads * g.d;
    const cuuint64_t dims[4] = {C, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.B};
    const cuuint64_t strides[3] = {C * 2, C * 2 * g.W, C * 2 * g.W * g.H};
    const cuuint32_t box[4] = {(cuuint32_t)g.d, (cuuint32_t)bw, (cuuint32_t)rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, g.d == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map of the factor table [heads][2][N][rank] as rows of rank values,
// box (rank, rows).
bool encode_factor_map(CUtensorMap *m, const void *base, const Geometry &g, int rows)
{
    auto fn = tensor_map_encoder();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)g.rank, (cuuint64_t)g.heads * 2 * g.N};
    const cuuint64_t strides[1] = {(cuuint64_t)g.rank * 2};
    const cuuint32_t box[2] = {(cuuint32_t)g.rank, (cuuint32_t)rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, g.rank == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether the built large-window kernel has exactly kLargeRegsLaunch
// registers per thread: its warpgroups' setmaxnreg shares add up to the
// launch's registers only then.  Looked up once per instantiation.
template <int D, int R, int BN, bool PAD>
bool large_regs_ok()
{
    static const bool ok = [] {
        cudaFuncAttributes fa;
        return cudaFuncGetAttributes(&fa, winattn_fwd_large_kernel<D, R, BN, PAD>) == cudaSuccess &&
               fa.numRegs == (int)kLargeRegsLaunch;
    }();
    return ok;
}

template <int D, int R, int BN, bool PAD>
int launch_large(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
                 float *lse, const Geometry &g, cudaStream_t stream)
{
    using T = __nv_bfloat16;
    // a build whose register count differs would wait forever in setmaxnreg:
    // its problems go to the generic tensor-core kernel instead
    if (!large_regs_ok<D, R, BN, PAD>())
        return launch_tc<D, R>(q, k, v, theta, bias, out, lse, g, stream);
    MapSet ms;
    const MapKey key = make_key(kLarge, g, k, v, bias, nullptr, nullptr);
    const bool ok = cached_maps(key, &ms, [&](MapSet *m) {
        const int kr = BN / g.M;
        if (!encode_kv_map(&m->m[0], k, g, g.M, kr) || !encode_kv_map(&m->m[2], v, g, g.M, kr))
            return false;
        if (g.shift && (!encode_kv_map(&m->m[1], k, g, g.M / 2, kr) || !encode_kv_map(&m->m[3], v, g, g.M / 2, kr)))
            return false;
        return R == 0 || encode_factor_map(&m->m[4], bias, g, BN);
    });
    if (!ok)
        return WINATTN_ERR_CUDA;
    static_assert(sizeof(LargeMaps) == 5 * sizeof(CUtensorMap), "LargeMaps is five maps");
    LargeMaps maps;
    std::memcpy(&maps, ms.m, sizeof maps);
    auto kernel = winattn_fwd_large_kernel<D, R, BN, PAD>;
    if (!smem_attr_once<winattn_fwd_large_kernel<D, R, BN, PAD>>())
        return WINATTN_ERR_CUDA;
    // all 512 TMEM columns per CTA: enough shared memory that no second CTA
    // is resident on the same SM
    const int need = (int)LargeLayout<D, R, BN>::BYTES;
    const int smem = need > 116 * 1024 ? need : 116 * 1024;
    const int64_t items = g.wph * g.heads * (g.N / 256);
    const int64_t grid = items < sm_count() ? items : sm_count();
    kernel<<<(unsigned)grid, kLargeThreads, smem, stream>>>(static_cast<const T *>(q), theta,
                                                           static_cast<const T *>(bias), static_cast<T *>(out), lse,
                                                           g, 1.0f / std::sqrt((float)g.d), maps);
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

template <int D, int R>
int launch_large_bn(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
                    float *lse, const Geometry &g, cudaStream_t s)
{
    if (large_tile_keys(g.M) == 96)
        return g.padded ? launch_large<D, R, 96, true>(q, k, v, theta, bias, out, lse, g, s)
                        : launch_large<D, R, 96, false>(q, k, v, theta, bias, out, lse, g, s);
    return g.padded ? launch_large<D, R, 128, true>(q, k, v, theta, bias, out, lse, g, s)
                    : launch_large<D, R, 128, false>(q, k, v, theta, bias, out, lse, g, s);
}

template <int D, int R, bool TMA>
int launch_small_variant(const void *q, const void *k, const void *v, const float *theta, const void *bias,
                         void *out, const Geometry &g, cudaStream_t stream, const WindowMaps *maps)
{
    using T = __nv_bfloat16;
    auto kernel = winattn_fwd_small_kernel<D, R, TMA>;
    // The kernel takes all 512 TMEM columns: ask for enough shared memory that
    // no second CTA can be resident on the same SM.
    const int need = (int)SmallLayout<D, R>::bytes(g.heads, g.M);
    const int smem = need > 116 * 1024 ? need : 116 * 1024;
    if (!smem_attr_once<winattn_fwd_small_kernel<D, R, TMA>>())
        return WINATTN_ERR_CUDA;
    const int64_t grid = g.items < sm_count() ? g.items : sm_count();
    kernel<<<(unsigned)grid, SmallRoles<D>::kThreads, smem, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), theta,
        static_cast<const T *>(bias), static_cast<T *>(out), g, 1.0f / std::sqrt((float)g.d), maps[0], maps[1],
        maps[2]);
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

template <int D, int R>
int launch_small(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
                 const Geometry &g, cudaStream_t stream)
{
    WindowMaps maps[3];
    std::memset(maps, 0, sizeof maps);
    if constexpr (R == 0) {
        if (small_tma_ok(g)) {
            MapSet ms;
            const MapKey key = make_key(kSmall, g, q, k, v, nullptr, nullptr);
            if (cached_maps(key, &ms, [&](MapSet *m) {
                    WindowMaps *w = reinterpret_cast<WindowMaps *>(m->m);
                    return encode_window_maps(&w[0], q, g) && encode_window_maps(&w[1], k, g) &&
                           encode_window_maps(&w[2], v, g);
                })) {
                std::memcpy(maps, ms.m, sizeof maps);
                return launch_small_variant<D, R, true>(q, k, v, theta, bias, out, g, stream, maps);
            }
            std::memset(maps, 0, sizeof maps);
        }
    }
    return launch_small_variant<D, R, false>(q, k, v, theta, bias, out, g, stream, maps);
}

template <int D>
int launch_pipe(const void *q, const void *k, const void *v, const float *theta, void *out, float *lse,
                const Geometry &g, cudaStream_t stream)
{
    static_assert(sizeof(WindowMaps) == 4 * sizeof(CUtensorMap), "WindowMaps is four maps");
    MapSet ms;
    const MapKey key = make_key(kPipe, g, q, k, v, out, nullptr);
    if (!cached_maps(key, &ms, [&](MapSet *m) {
            WindowMaps *w = reinterpret_cast<WindowMaps *>(m->m);
            return encode_window_maps(&w[0], q, g) && encode_window_maps(&w[1], k, g) &&
                   encode_window_maps(&w[2], v, g) && encode_window_maps(&w[3], out, g);
        }))
        return WINATTN_ERR_CUDA;
    WindowMaps maps[4];
    std::memcpy(maps, ms.m, sizeof maps);
    auto kernel = winattn_fwd_pipe_kernel<D>;
    const int smem = (int)PipeLayout<D>::bytes(g.heads);
    if (!smem_attr_once<winattn_fwd_pipe_kernel<D>>())
        return WINATTN_ERR_CUDA;
    const int64_t grid = g.items < sm_count() ? g.items : sm_count();
    // a programmatic dependent of the previous kernel in the stream: its
    // launch and prologue overlap that kernel's tail (the kernel waits for it
    // before touching global memory)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPipeThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float scale = 1.0f / std::sqrt((float)g.d);
    if (cudaLaunchKernelEx(&cfg, kernel, theta, static_cast<__nv_bfloat16 *>(out), lse, g, scale, maps[0], maps[1],
                           maps[2], maps[3]) != cudaSuccess)
        return WINATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

template <int D>
int launch_pipe16(const void *q, const void *k, const void *v, const float *theta, void *out, float *lse,
                  const Geometry &g, cudaStream_t stream)
{
    static_assert(sizeof(Pipe16StoreMaps) == 2 * sizeof(CUtensorMap), "two store maps");
    MapSet ms;
    const MapKey key = make_key(kPipe16, g, q, k, v, out, nullptr);
    if (!cached_maps(key, &ms, [&](MapSet *m) {
            WindowMaps *w = reinterpret_cast<WindowMaps *>(m->m);
            return encode_window_maps(&w[0], q, g) && encode_window_maps(&w[1], k, g) &&
                   encode_window_maps(&w[2], v, g) && encode_window_map(&m->m[12], out, g, 16, 2) &&
                   encode_window_map(&m->m[13], out, g, 8, 4);
        }))
        return WINATTN_ERR_CUDA;
    WindowMaps maps[3];
    Pipe16StoreMaps om;
    std::memcpy(maps, ms.m, sizeof maps);
    std::memcpy(&om, &ms.m[12], sizeof om);
    if (!smem_attr_once<winattn_fwd_pipe16_kernel<D>>())
        return WINATTN_ERR_CUDA;
    const int smem = (int)Pipe16Layout<D>::bytes(g.heads);
    const int64_t items = g.wph * g.heads;
    const int64_t grid = items < sm_count() ? items : sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kP16Threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float scale = 1.0f / std::sqrt((float)g.d);
    if (cudaLaunchKernelEx(&cfg, winattn_fwd_pipe16_kernel<D>, theta, lse, g, scale, maps[0], maps[1], maps[2], om) !=
        cudaSuccess)
        return WINATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

template <int D, int R>
int launch_simt(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
                float *lse, const Geometry &g, cudaStream_t stream)
{
    return launch<winattn_fwd_simt_kernel<D, R>>((int)SimtLayout<D, R>::bytes(g.M), g, stream,
                  static_cast<const float *>(q), static_cast<const float *>(k), static_cast<const float *>(v),
                  theta, static_cast<const float *>(bias), static_cast<float *>(out), lse);
}

int dispatch(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
             const Geometry &g, int dtype, cudaStream_t s, float *lse = nullptr)
{
    const KernelKind kind = choose_kernel(g, dtype, lse != nullptr);
    if (kind == kPipe)
        return g.d == 32 ? launch_pipe<32>(q, k, v, theta, out, lse, g, s)
                         : launch_pipe<64>(q, k, v, theta, out, lse, g, s);
    if (kind == kPipe16)
        return g.d == 32 ? launch_pipe16<32>(q, k, v, theta, out, lse, g, s)
                         : launch_pipe16<64>(q, k, v, theta, out, lse, g, s);
    if (kind == kSmall) {
        switch (g.d * 100 + g.rank) {
        case 3200: return launch_small<32, 0>(q, k, v, theta, bias, out, g, s);
        case 3216: return launch_small<32, 16>(q, k, v, theta, bias, out, g, s);
        case 3232: return launch_small<32, 32>(q, k, v, theta, bias, out, g, s);
        case 6400: return launch_small<64, 0>(q, k, v, theta, bias, out, g, s);
        case 6416: return launch_small<64, 16>(q, k, v, theta, bias, out, g, s);
        case 6432: return launch_small<64, 32>(q, k, v, theta, bias, out, g, s);
        }
    } else if (kind == kLarge) {
        switch (g.d * 100 + g.rank) {
        case 3200: return launch_large_bn<32, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 3216: return launch_large_bn<32, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 3232: return launch_large_bn<32, 32>(q, k, v, theta, bias, out, lse, g, s);
        case 6400: return launch_large_bn<64, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 6416: return launch_large_bn<64, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 6432: return launch_large_bn<64, 32>(q, k, v, theta, bias, out, lse, g, s);
        }
    } else if (kind == kGeneric) {
        switch (g.d * 100 + g.rank) {
        case 3200: return launch_tc<32, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 3216: return launch_tc<32, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 3232: return launch_tc<32, 32>(q, k, v, theta, bias, out, lse, g, s);
        case 6400: return launch_tc<64, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 6416: return launch_tc<64, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 6432: return launch_tc<64, 32>(q, k, v, theta, bias, out, lse, g, s);
        }
    } else {
        switch (g.d * 100 + g.rank) {
        case 1600: return launch_simt<16, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 1616: return launch_simt<16, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 1632: return launch_simt<16, 32>(q, k, v, theta, bias, out, lse, g, s);
        case 3200: return launch_simt<32, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 3216: return launch_simt<32, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 3232: return launch_simt<32, 32>(q, k, v, theta, bias, out, lse, g, s);
        case 6400: return launch_simt<64, 0>(q, k, v, theta, bias, out, lse, g, s);
        case 6416: return launch_simt<64, 16>(q, k, v, theta, bias, out, lse, g, s);
        case 6432: return launch_simt<64, 32>(q, k, v, theta, bias, out, lse, g, s);
        }
    }
    return WINATTN_ERR_ARG;
}

// Streams and events of the host-buffer entry points, created once per device
// (with that device current) and kept until the process exits; a mutex per
// device keeps concurrent host-buffer calls from interleaving their records.
constexpr int kHostLanes = 3, kHostChunks = 8;

struct HostLanes {
    std::mutex mu;
    cudaStream_t lane[kHostLanes];
    cudaEvent_t entry, done[kHostLanes];
};

HostLanes *host_lanes()
{
    static std::mutex mu;
    static HostLanes *per_dev[64];
    const int dev = current_device();
    if (dev < 0)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!per_dev[dev]) {
        HostLanes *h = new HostLanes;
        bool ok = cudaEventCreateWithFlags(&h->entry, cudaEventDisableTiming) == cudaSuccess;
        for (int l = 0; ok && l < kHostLanes; ++l)
            ok = cudaStreamCreateWithFlags(&h->lane[l], cudaStreamNonBlocking) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h->done[l], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            delete h;  // the handles created so far stay with the context
            return nullptr;
        }
        per_dev[dev] = h;
    }
    return per_dev[dev];
}

// ------------------------------------------------------------------ gated windows

template <int D, int R>
int launch_sparse(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
                  const int32_t *windows, int n_windows, const Geometry &g, cudaStream_t stream)
{
    using T = __nv_bfloat16;
    constexpr auto kernel = winattn_fwd_tc_kernel<D, R, true>;
    if (!smem_attr_once<kernel>())
        return WINATTN_ERR_CUDA;
    const int64_t items = (int64_t)g.heads * ((n_windows + g.U - 1) / g.U) * g.n_tiles;
    kernel<<<(unsigned)items, kThreads, TcLayout<D, R, true>::bytes(g.M), stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), theta,
        static_cast<const T *>(bias), static_cast<T *>(out), nullptr, g, 1.0f / std::sqrt((float)g.d), windows,
        n_windows);
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

int dispatch_sparse(const void *q, const void *k, const void *v, const float *theta, const void *bias, void *out,
                    const int32_t *windows, int n_windows, const Geometry &g, cudaStream_t s)
{
    switch (g.d * 100 + g.rank) {
    case 3200: return launch_sparse<32, 0>(q, k, v, theta, bias, out, windows, n_windows, g, s);
    case 3216: return launch_sparse<32, 16>(q, k, v, theta, bias, out, windows, n_windows, g, s);
    case 3232: return launch_sparse<32, 32>(q, k, v, theta, bias, out, windows, n_windows, g, s);
    case 6400: return launch_sparse<64, 0>(q, k, v, theta, bias, out, windows, n_windows, g, s);
    case 6416: return launch_sparse<64, 16>(q, k, v, theta, bias, out, windows, n_windows, g, s);
    case 6432: return launch_sparse<64, 32>(q, k, v, theta, bias, out, windows, n_windows, g, s);
    }
    return WINATTN_ERR_ARG;
}

// ------------------------------------------------------------------ backward

struct BwdArgs {
    const void *q, *k, *v;
    const float *theta;
    const void *bias, *out, *dout;
    const float *lse;
    void *dq, *dk, *dv;
    float *dtheta, *dbias, *dq_acc;
};

template <int D, int R>
int launch_bwd(const BwdArgs &a, const Geometry &g, cudaStream_t s)
{
    using T = __nv_bfloat16;
    const int smem = (int)BwdLayout<D, R>::bytes(g.M);
    if (!smem_attr_once<winattn_bwd_tc_kernel<D, R>>())
        return WINATTN_ERR_CUDA;
    const float scale = 1.0f / std::sqrt((float)g.d);
    winattn_bwd_tc_kernel<D, R><<<(unsigned)g.items, kBwdThreads, smem, s>>>(
        static_cast<const T *>(a.q), static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.theta,
        static_cast<const T *>(a.bias), static_cast<const T *>(a.out), static_cast<const T *>(a.dout), a.lse,
        static_cast<T *>(a.dq), static_cast<T *>(a.dk), static_cast<T *>(a.dv), a.dtheta, a.dbias, a.dq_acc, g,
        scale);
    if (cudaGetLastError() != cudaSuccess)
        return WINATTN_ERR_CUDA;
    if (g.n_tiles > 1) {
        const int64_t T_tok = (int64_t)g.B * g.H * g.W;
        const dim3 grid((unsigned)((T_tok + 127) / 128), (unsigned)g.heads);
        winattn_bwd_finalize_kernel<D><<<grid, 128, 0, s>>>(static_cast<const T *>(a.q), a.theta, a.dq_acc,
                                                            static_cast<T *>(a.dq), a.dtheta, g, scale);
        if (cudaGetLastError() != cudaSuccess)
            return WINATTN_ERR_CUDA;
    }
    return WINATTN_OK;
}

int dispatch_bwd(const BwdArgs &a, const Geometry &g, cudaStream_t s)
{
    switch (g.d * 100 + g.rank) {
    case 3200: return launch_bwd<32, 0>(a, g, s);
    case 3216: return launch_bwd<32, 16>(a, g, s);
    case 3232: return launch_bwd<32, 32>(a, g, s);
    case 6400: return launch_bwd<64, 0>(a, g, s);
    case 6416: return launch_bwd<64, 16>(a, g, s);
    case 6432: return launch_bwd<64, 32>(a, g, s);
    }
    return WINATTN_ERR_ARG;
}

}  // namespace
}  // namespace winattn

using namespace winattn;

extern "C" {

int winattn_check_args(const void *q, const void *k, const void *v, const float *theta, const void *bias_feats,
                       int B, int H_img, int W_img, int M, int shift, int heads, int d, int rank, int dtype,
                       const void *out)
{
    const int rc = check_sizes(B, H_img, W_img, M, shift, heads, d, rank, dtype);
    if (rc != WINATTN_OK)
        return rc;
    if (!q || !k || !v || !out)
        return WINATTN_ERR_ARG;
    if ((rank > 0) != (bias_feats != nullptr))
        return WINATTN_ERR_RANK;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (bias_feats && !aligned16(bias_feats)) || (reinterpret_cast<uintptr_t>(theta) & 3u))
        return WINATTN_ERR_ALIGN;
    const size_t n = map_bytes(B, H_img, W_img, heads, d, dtype);
    if (overlaps(out, n, q, n) || overlaps(out, n, k, n) || overlaps(out, n, v, n))
        return WINATTN_ERR_ALIAS;
    return WINATTN_OK;
}

int winattn_fwd(const void *q, const void *k, const void *v, const float *theta, const void *bias_feats, int B,
                int H_img, int W_img, int M, int shift, int heads, int d, int rank, int dtype, void *out,
                void *stream)
{
    int rc = winattn_check_args(q, k, v, theta, bias_feats, B, H_img, W_img, M, shift, heads, d, rank, dtype, out);
    if (rc != WINATTN_OK)
        return rc;
    rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    const Geometry g = Geometry::make(B, H_img, W_img, M, shift, heads, d, rank);
    return dispatch(q, k, v, theta, bias_feats, out, g, dtype, static_cast<cudaStream_t>(stream));
}

int winattn_fwd_sparse(const void *q, const void *k, const void *v, const float *theta, const void *bias_feats,
                       int B, int H_img, int W_img, int M, int shift, int heads, int d, int rank, int dtype,
                       const int32_t *windows, int n_windows, void *out, void *stream)
{
    // out holds O_lin and is updated in place: it may not alias q, k, v
    int rc = winattn_check_args(q, k, v, theta, bias_feats, B, H_img, W_img, M, shift, heads, d, rank, dtype, out);
    if (rc != WINATTN_OK)
        return rc;
    if (dtype != WINATTN_BF16)
        return WINATTN_ERR_DTYPE;
    if (n_windows < 0 || (n_windows > 0 && !windows))
        return WINATTN_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(windows) & 3u)
        return WINATTN_ERR_ALIGN;
    if (n_windows == 0)
        return WINATTN_OK;
    rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    const Geometry g = Geometry::make(B, H_img, W_img, M, shift, heads, d, rank);
    if (n_windows > g.wph)
        return WINATTN_ERR_ARG;  // windows may not repeat, so at most every window once
    return dispatch_sparse(q, k, v, theta, bias_feats, out, windows, n_windows, g, static_cast<cudaStream_t>(stream));
}

int winattn_rib_features(const float *w1, const float *w2, int M, int heads, int rank, void *table, void *stream)
{
    if (!w1 || !w2 || !table || M <= 0 || M > kMaxM || heads <= 0)
        return WINATTN_ERR_ARG;
    if (rank != 16 && rank != 32)
        return WINATTN_ERR_RANK;
    if (!aligned16(table) || !aligned16(w1) || !aligned16(w2))
        return WINATTN_ERR_ALIGN;
    const int rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    const dim3 grid((unsigned)((M * M + 127) / 128), (unsigned)(heads * 2));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto *t = static_cast<__nv_bfloat16 *>(table);
    if (rank == 16)
        winattn_rib_features_kernel<16><<<grid, 128, 0, s>>>(w1, w2, M, t);
    else
        winattn_rib_features_kernel<32><<<grid, 128, 0, s>>>(w1, w2, M, t);
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

int winattn_fwd_rib(const void *q, const void *k, const void *v, const float *theta, const float *w1, const float *w2,
                    int B, int H_img, int W_img, int M, int shift, int heads, int d, int rank, int dtype, void *table,
                    void *out, void *stream)
{
    if (dtype != WINATTN_BF16)
        return WINATTN_ERR_DTYPE;
    if (!table)
        return WINATTN_ERR_ARG;
    // every argument of the attention is checked before the table is written
    int rc = winattn_check_args(q, k, v, theta, table, B, H_img, W_img, M, shift, heads, d, rank, dtype, out);
    if (rc != WINATTN_OK)
        return rc;
    const size_t nt = (size_t)heads * 2 * M * M * rank * 2, n = map_bytes(B, H_img, W_img, heads, d, dtype);
    if (overlaps(table, nt, q, n) || overlaps(table, nt, k, n) || overlaps(table, nt, v, n) ||
        overlaps(table, nt, out, n))
        return WINATTN_ERR_ALIAS;
    rc = winattn_rib_features(w1, w2, M, heads, rank, table, stream);
    if (rc != WINATTN_OK)
        return rc;
    return winattn_fwd(q, k, v, theta, table, B, H_img, W_img, M, shift, heads, d, rank, dtype, out, stream);
}

int winattn_cla_gate(const void *x, const void *o, const float *dw, const float *dw_b, const float *pw,
                     const float *pw_b, int B, int H_img, int W_img, int C, int dtype, void *out, void *stream)
{
    if (dtype != WINATTN_BF16)
        return WINATTN_ERR_DTYPE;
    if (!x || !o || !dw || !dw_b || !pw || !pw_b || !out || B <= 0 || H_img <= 0 || W_img <= 0)
        return WINATTN_ERR_ARG;
    if (C < 16 || C > 256 || C % 16)
        return WINATTN_ERR_ARG;
    if (!aligned16(x) || !aligned16(o) || !aligned16(out) || (reinterpret_cast<uintptr_t>(dw) & 3u) ||
        (reinterpret_cast<uintptr_t>(dw_b) & 3u) || (reinterpret_cast<uintptr_t>(pw) & 3u) ||
        (reinterpret_cast<uintptr_t>(pw_b) & 3u))
        return WINATTN_ERR_ALIGN;
    const size_t n = (size_t)B * H_img * W_img * C * 2;
    if (overlaps(out, n, x, n) || (out != o && overlaps(out, n, o, n)))
        return WINATTN_ERR_ALIAS;
    const int rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    if (!smem_attr_once<winattn_cla_gate_kernel>())
        return WINATTN_ERR_CUDA;
    const int64_t tiles = ((int64_t)B * H_img * W_img + 127) / 128;
    const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
    winattn_cla_gate_kernel<<<grid, kGateThreads, GateLayout::bytes(C), static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(o), dw, dw_b, pw, pw_b, B, H_img,
        W_img, C, static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

size_t winattn_bwd_workspace_bytes(int B, int H_img, int W_img, int M, int heads, int d)
{
    if (B <= 0 || H_img <= 0 || W_img <= 0 || M <= 0 || M > kMaxM || heads <= 0 || (d != 32 && d != 64))
        return 0;
    // windows of more than one 128-row tile sum dQ over their key tiles in fp32
    if ((int64_t)M * M <= kTileRows)
        return 0;
    return ((size_t)B * H_img * W_img * heads * d * 4 + 255) & ~size_t(255);
}

int winattn_bwd(const void *q, const void *k, const void *v, const float *theta, const void *bias_feats,
                const void *out, const void *dout, const float *lse, int B, int H_img, int W_img, int M, int shift,
                int heads, int d, int rank, int dtype, void *dq, void *dk, void *dv, float *dtheta, float *dbias,
                void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_sizes(B, H_img, W_img, M, shift, heads, d, rank, dtype);
    if (rc != WINATTN_OK)
        return rc;
    if (dtype != WINATTN_BF16)
        return WINATTN_ERR_DTYPE;
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv)
        return WINATTN_ERR_ARG;
    if ((rank > 0) != (bias_feats != nullptr))
        return WINATTN_ERR_RANK;
    if ((dtheta && !theta) || (dbias && !bias_feats))
        return WINATTN_ERR_ARG;
    const void *maps[8] = {q, k, v, out, dout, dq, dk, dv};
    for (const void *p : maps)
        if (!aligned16(p))
            return WINATTN_ERR_ALIGN;
    if ((bias_feats && !aligned16(bias_feats)) || (dbias && !aligned16(dbias)) ||
        (reinterpret_cast<uintptr_t>(theta) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
        (reinterpret_cast<uintptr_t>(dtheta) & 3u))
        return WINATTN_ERR_ALIGN;
    const size_t n = map_bytes(B, H_img, W_img, heads, d, dtype);
    // the three gradients must not overlap one another or any input map
    for (int o = 5; o < 8; ++o)
        for (int i = 0; i < 8; ++i)
            if (i != o && overlaps(maps[o], n, maps[i], n))
                return WINATTN_ERR_ALIAS;
    const size_t need = winattn_bwd_workspace_bytes(B, H_img, W_img, M, heads, d);
    if (need && (!workspace || workspace_bytes < need))
        return WINATTN_ERR_SIZE;
    if (need && !aligned16(workspace))
        return WINATTN_ERR_ALIGN;
    rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Geometry g = Geometry::make(B, H_img, W_img, M, shift, heads, d, rank);
    // the theta and bias-table gradients and the dQ sums are accumulated
    if ((dtheta && cudaMemsetAsync(dtheta, 0, (size_t)heads * (d / 4) * 4, s) != cudaSuccess) ||
        (dbias && cudaMemsetAsync(dbias, 0, (size_t)heads * 2 * g.N * rank * 4, s) != cudaSuccess) ||
        (need && cudaMemsetAsync(workspace, 0, need, s) != cudaSuccess))
        return WINATTN_ERR_CUDA;
    BwdArgs a{q, k, v, theta, bias_feats, out, dout, lse, dq, dk, dv, dtheta, dbias,
              need ? static_cast<float *>(workspace) : nullptr};
    return dispatch_bwd(a, g, s);
}

int winattn_fwd_lse(const void *q, const void *k, const void *v, const float *theta, const void *bias_feats, int B,
                    int H_img, int W_img, int M, int shift, int heads, int d, int rank, int dtype, void *out, float *lse,
                    void *stream)
{
    int rc = winattn_check_args(q, k, v, theta, bias_feats, B, H_img, W_img, M, shift, heads, d, rank, dtype, out);
    if (rc != WINATTN_OK)
        return rc;
    if (!lse)
        return WINATTN_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(lse) & 3u)
        return WINATTN_ERR_ALIGN;
    const size_t n = map_bytes(B, H_img, W_img, heads, d, dtype), nl = (size_t)B * H_img * W_img * heads * 4;
    if (overlaps(lse, nl, q, n) || overlaps(lse, nl, k, n) || overlaps(lse, nl, v, n) || overlaps(lse, nl, out, n))
        return WINATTN_ERR_ALIAS;
    rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    const Geometry g = Geometry::make(B, H_img, W_img, M, shift, heads, d, rank);
    return dispatch(q, k, v, theta, bias_feats, out, g, dtype, static_cast<cudaStream_t>(stream), lse);
}

size_t winattn_host_workspace_bytes(int B, int H_img, int W_img, int heads, int d, int dtype)
{
    if (B <= 0 || H_img <= 0 || W_img <= 0 || heads <= 0 || d <= 0 ||
        (dtype != WINATTN_BF16 && dtype != WINATTN_FP32))
        return 0;
    const size_t n = (map_bytes(B, H_img, W_img, heads, d, dtype) + 255) & ~size_t(255);
    return 4 * n;
}

}  // extern "C"

namespace {

// The host-buffer call.  With `overlap`, the batch is cut into chunks of
// whole images (a window never spans two images, so each chunk is an exact
// sub-problem) that take turns on the library's lanes, so that one chunk's
// kernel and read-back overlap the next chunk's upload (host-to-device and
// device-to-host copies run on separate copy engines); without it, copies and
// kernel are enqueued on the caller's stream alone.
int fwd_host_impl(const void *q_host, const void *k_host, const void *v_host, const float *theta,
                  const void *bias_feats, int B, int H_img, int W_img, int M, int shift, int heads, int d, int rank,
                  int dtype, void *out_host, void *workspace, size_t workspace_bytes, void *stream, bool overlap)
{
    int rc = check_sizes(B, H_img, W_img, M, shift, heads, d, rank, dtype);
    if (rc != WINATTN_OK)
        return rc;
    if (!q_host || !k_host || !v_host || !out_host || !workspace)
        return WINATTN_ERR_ARG;
    if (workspace_bytes < winattn_host_workspace_bytes(B, H_img, W_img, heads, d, dtype))
        return WINATTN_ERR_SIZE;
    if (!aligned16(workspace))
        return WINATTN_ERR_ALIGN;
    const size_t n = map_bytes(B, H_img, W_img, heads, d, dtype);
    const size_t stride = (n + 255) & ~size_t(255);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *dq = ws, *dk = ws + stride, *dv = ws + 2 * stride, *dout = ws + 3 * stride;
    rc = winattn_check_args(dq, dk, dv, theta, bias_feats, B, H_img, W_img, M, shift, heads, d, rank, dtype, dout);
    if (rc != WINATTN_OK)
        return rc;
    rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!overlap) {
        if (cudaMemcpyAsync(dq, q_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(dk, k_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(dv, v_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return WINATTN_ERR_CUDA;
        const Geometry g = Geometry::make(B, H_img, W_img, M, shift, heads, d, rank);
        rc = dispatch(dq, dk, dv, theta, bias_feats, dout, g, dtype, s);
        if (rc != WINATTN_OK)
            return rc;
        return cudaMemcpyAsync(out_host, dout, n, cudaMemcpyDeviceToHost, s) == cudaSuccess ? WINATTN_OK
                                                                                           : WINATTN_ERR_CUDA;
    }
    HostLanes *lanes = host_lanes();
    if (!lanes)
        return WINATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(lanes->mu);
    const int chunks = B < kHostChunks ? B : kHostChunks;
    const size_t img = n / (size_t)B;
    if (cudaEventRecord(lanes->entry, s) != cudaSuccess)
        return WINATTN_ERR_CUDA;
    for (int l = 0; l < kHostLanes && l < chunks; ++l)
        if (cudaStreamWaitEvent(lanes->lane[l], lanes->entry, 0) != cudaSuccess)
            return WINATTN_ERR_CUDA;
    int b0 = 0;
    for (int c = 0; c < chunks; ++c) {
        const int nb = B / chunks + (c < B % chunks ? 1 : 0);
        const size_t off = (size_t)b0 * img, len = (size_t)nb * img;
        cudaStream_t ls = lanes->lane[c % kHostLanes];
        const uint8_t *hq = static_cast<const uint8_t *>(q_host) + off;
        const uint8_t *hk = static_cast<const uint8_t *>(k_host) + off;
        const uint8_t *hv = static_cast<const uint8_t *>(v_host) + off;
        if (cudaMemcpyAsync(dq + off, hq, len, cudaMemcpyHostToDevice, ls) != cudaSuccess ||
            cudaMemcpyAsync(dk + off, hk, len, cudaMemcpyHostToDevice, ls) != cudaSuccess ||
            cudaMemcpyAsync(dv + off, hv, len, cudaMemcpyHostToDevice, ls) != cudaSuccess)
            return WINATTN_ERR_CUDA;
        const Geometry g = Geometry::make(nb, H_img, W_img, M, shift, heads, d, rank);
        rc = dispatch(dq + off, dk + off, dv + off, theta, bias_feats, dout + off, g, dtype, ls);
        if (rc != WINATTN_OK)
            return rc;
        if (cudaMemcpyAsync(static_cast<uint8_t *>(out_host) + off, dout + off, len, cudaMemcpyDeviceToHost, ls) !=
            cudaSuccess)
            return WINATTN_ERR_CUDA;
        b0 += nb;
    }
    // the caller's stream resumes once every lane has finished its chunks
    for (int l = 0; l < kHostLanes && l < chunks; ++l)
        if (cudaEventRecord(lanes->done[l], lanes->lane[l]) != cudaSuccess ||
            cudaStreamWaitEvent(s, lanes->done[l], 0) != cudaSuccess)
            return WINATTN_ERR_CUDA;
    return WINATTN_OK;
}

}  // namespace

extern "C" {

int winattn_fwd_host(const void *q_host, const void *k_host, const void *v_host, const float *theta,
                     const void *bias_feats, int B, int H_img, int W_img, int M, int shift, int heads, int d,
                     int rank, int dtype, void *out_host, void *workspace, size_t workspace_bytes, void *stream)
{
    return fwd_host_impl(q_host, k_host, v_host, theta, bias_feats, B, H_img, W_img, M, shift, heads, d, rank,
                         dtype, out_host, workspace, workspace_bytes, stream, true);
}

}  // extern "C"

namespace {

// Library-owned device workspace of winattn_fwd_host_static (the device copies
// of q, k, v and out).  In host code the name stands for a host-side shadow,
// not a device address: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_static_workspace[WINATTN_STATIC_WORKSPACE_BYTES];

// Device address of g_static_workspace on the current device, looked up once
// per device with that device current; nullptr if the lookup failed.
void *static_workspace_ptr()
{
    static std::mutex mu;
    static void *cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cached[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess)
            return nullptr;
        cached[dev] = ptr;
    }
    return cached[dev];
}

}  // namespace

namespace winattn {

// One warp waits on an mbarrier that nothing arrives at, through the same
// bounded wait every persistent kernel uses: the wait must give up after its
// time limit, set the CTA's abort flag and the device status word, and
// return, so the context stays usable.
__global__ void selftest_wait_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_word;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_word = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    warp_wait(&bar, 0, &abort_word);
}

}  // namespace winattn

extern "C" {

int winattn_fwd_host_static(const void *q_host, const void *k_host, const void *v_host, const float *theta,
                            const void *bias_feats, int B, int H_img, int W_img, int M, int shift, int heads, int d,
                            int rank, int dtype, void *out_host, void *stream)
{
    const int rc = check_sizes(B, H_img, W_img, M, shift, heads, d, rank, dtype);
    if (rc != WINATTN_OK)
        return rc;
    const size_t need = winattn_host_workspace_bytes(B, H_img, W_img, heads, d, dtype);
    if (need == 0 || need > WINATTN_STATIC_WORKSPACE_BYTES)
        return WINATTN_ERR_SIZE;
    const int dev_rc = check_device();
    if (dev_rc != WINATTN_OK)
        return dev_rc;
    void *ws = static_workspace_ptr();
    if (!ws)
        return WINATTN_ERR_CUDA;
    return fwd_host_impl(q_host, k_host, v_host, theta, bias_feats, B, H_img, W_img, M, shift, heads, d, rank,
                         dtype, out_host, ws, WINATTN_STATIC_WORKSPACE_BYTES, stream, false);
}

const char *winattn_strerror(int code)
{
    switch (code) {
    case WINATTN_OK: return "success";
    case WINATTN_ERR_ARG: return "invalid argument (null pointer, size, window/map mismatch, shift or head dim)";
    case WINATTN_ERR_RANK: return "bias rank and bias_feats pointer disagree, or unsupported rank";
    case WINATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
    case WINATTN_ERR_DTYPE: return "unsupported dtype";
    case WINATTN_ERR_ARCH: return "device is not compute capability 10.0 (B200, sm_100a)";
    case WINATTN_ERR_CUDA: return "CUDA runtime error or kernel launch failure";
    case WINATTN_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case WINATTN_ERR_ALIAS: return "out overlaps q, k or v";
    case WINATTN_ERR_SIZE: return "problem too large for the index range, or workspace too small";
    case WINATTN_ERR_DEVICE_BOUNDS: return "a debug build found an index or TMA box outside the map";
    }
    return "unknown error code";
}

int winattn_last_device_status(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return WINATTN_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof word) != cudaSuccess)
        return WINATTN_ERR_CUDA;
    if (word) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero) != cudaSuccess)
            return WINATTN_ERR_CUDA;
        return (word & 1u) ? WINATTN_ERR_DEVICE_TIMEOUT : WINATTN_ERR_DEVICE_BOUNDS;
    }
    return WINATTN_OK;
}

int winattn_launch_info(int B, int H_img, int W_img, int M, int shift, int heads, int d, int rank, int dtype,
                        int64_t *work_items, int *grid, int *threads, int *smem_bytes, int *windows_per_tile,
                        int *kernel)
{
    const int rc = check_sizes(B, H_img, W_img, M, shift, heads, d, rank, dtype);
    if (rc != WINATTN_OK)
        return rc;
    const Geometry g = Geometry::make(B, H_img, W_img, M, shift, heads, d, rank);
    const KernelKind kind = choose_kernel(g, dtype);
    if (work_items) *work_items = g.items;
    if (windows_per_tile) *windows_per_tile = g.U;
    if (kernel) *kernel = (int)kind;
    if (kind == kLarge) {
        const int64_t items = g.wph * g.heads * (g.N / 256);
        if (work_items) *work_items = items;
        if (grid) *grid = (int)(items < kAssumedSMs ? items : kAssumedSMs);
        if (threads) *threads = kLargeThreads;
        if (smem_bytes) *smem_bytes = (int)large_smem(g);
    } else if (kind == kPipe) {
        if (grid) *grid = (int)(g.items < kAssumedSMs ? g.items : kAssumedSMs);
        if (threads) *threads = kPipeThreads;
        if (smem_bytes) *smem_bytes = (int)pipe_smem(g);
    } else if (kind == kPipe16) {
        const int64_t items = g.wph * g.heads;  // window-heads: two query tiles each
        if (work_items) *work_items = items;
        if (grid) *grid = (int)(items < kAssumedSMs ? items : kAssumedSMs);
        if (threads) *threads = kP16Threads;
        if (smem_bytes) *smem_bytes = (int)pipe16_smem(g);
    } else if (kind == kSmall) {
        if (grid) *grid = (int)(g.items < kAssumedSMs ? g.items : kAssumedSMs);
        if (threads) *threads = g.d <= 32 ? SmallRoles<32>::kThreads : SmallRoles<64>::kThreads;
        if (smem_bytes) *smem_bytes = (int)small_smem(g);
    } else {
        if (grid) *grid = (int)g.items;
        if (threads) *threads = kThreads;
        if (smem_bytes) *smem_bytes = smem_bytes_for(g, dtype);
    }
    return WINATTN_OK;
}

int winattn_selftest_wait_timeout(void *stream)
{
    const int rc = check_device();
    if (rc != WINATTN_OK)
        return rc;
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    return cudaGetLastError() == cudaSuccess ? WINATTN_OK : WINATTN_ERR_CUDA;
}

int winattn_set_kernel_enabled(int kernel, int enabled)
{
    if (kernel != kSmall && kernel != kLarge && kernel != kPipe && kernel != kPipe16)
        return WINATTN_ERR_ARG;
    return g_kernel_enabled[kernel].exchange(enabled ? 1 : 0);
}

}  // extern "C"
