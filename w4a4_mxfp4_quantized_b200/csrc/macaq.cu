// macaq.cu -- the C ABI of libmacaq.so (declared in include/macaq.h): argument validation,
// tensor-map descriptors (cached), and the launches of the quantization and GEMM kernels.
//
// Everything is one translation unit so that the device status word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "macaq.h"
#include "flip.cuh"
#include "gemm.cuh"
#include "moe.cuh"
#include "quant.cuh"
#include "w4a16.cuh"

namespace macaq {

namespace {

constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitNs};
thread_local int t_last_cuda_error = 0;

macaq_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return MACAQ_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_block(int32_t b) { return b == 1 || b == 16 || b == 32 || b == 64 || b == 128; }

// ------------------------------------------------------------------------ device properties
struct DeviceInfo {
    int sms = 0;
    int major = 0;
    int minor = 0;
};

macaq_status device_info(DeviceInfo *out) {
    static std::mutex mu;
    static std::map<int, DeviceInfo> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it == cache.end()) {
        DeviceInfo d;
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
            return cuda_fail(e);
        it = cache.emplace(dev, d).first;
    }
    *out = it->second;
    if (out->major != 10) return MACAQ_ERR_UNSUPPORTED;  // built for sm_100a only
    return MACAQ_OK;
}

// ------------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

using MapKey = std::tuple<int, uintptr_t, int, int, std::array<uint64_t, 5>, std::array<uint64_t, 4>,
                          std::array<uint32_t, 5>, int>;

// A tiled tensor map of rank 2 to 5 over a strided array: dims[0] contiguous elements, dims[i] with
// byte stride strides[i-1]; box of box[0] x ... elements; zero fill out of bounds. Descriptors are
// cached by everything they encode.
macaq_status tensor_map(CUtensorMap *out, const void *base, CUtensorMapDataType dtype, int rank,
                        const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                        CUtensorMapSwizzle swizzle) {
    static std::mutex mu;
    static std::map<MapKey, CUtensorMap> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::array<uint64_t, 5> kd{};
    std::array<uint64_t, 4> ks{};
    std::array<uint32_t, 5> kb{};
    for (int i = 0; i < rank; ++i) {
        kd[i] = dims[i];
        kb[i] = box[i];
        if (i > 0) ks[i - 1] = strides[i - 1];
    }
    const MapKey key{dev, reinterpret_cast<uintptr_t>(base), static_cast<int>(dtype), rank, kd, ks, kb,
                     static_cast<int>(swizzle)};
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *out = it->second;
        return MACAQ_OK;
    }
    auto fn = encode_fn();
    if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
    CUtensorMap m;
    cuuint64_t d[5];
    cuuint64_t s[4];
    cuuint32_t b[5];
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        if (i > 0) s[i - 1] = strides[i - 1];
    }
    CUresult r = fn(&m, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d, s, b, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    if (cache.size() > 4096) cache.clear();
    cache.emplace(key, m);
    *out = m;
    return MACAQ_OK;
}

macaq_status tensor_map_2d(CUtensorMap *out, const void *base, CUtensorMapDataType dtype, uint64_t inner,
                           uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                           CUtensorMapSwizzle swizzle) {
    const uint64_t dims[2] = {inner, outer};
    const uint64_t strides[1] = {row_bytes};
    const uint32_t box[2] = {box_inner, box_outer};
    return tensor_map(out, base, dtype, 2, dims, strides, box, swizzle);
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device, size).
template <typename Kernel>
macaq_status set_smem(Kernel k, size_t bytes) {
    static std::mutex mu;
    static std::map<std::tuple<const void *, int>, size_t> done;
    int dev = 0;
    cudaGetDevice(&dev);
    const auto key = std::make_tuple(reinterpret_cast<const void *>(k), dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return MACAQ_OK;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e != cudaSuccess) return cuda_fail(e);
    done[key] = bytes;
    return MACAQ_OK;
}

// Every kernel is launched with programmatic stream serialization: it may start its prologue while
// the previous kernel in the stream finishes, and waits for that kernel (griddep_wait) before it
// touches memory the previous kernel may own. cluster > 1 adds the cluster shape.
template <typename Kernel, typename... Args>
macaq_status launch(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, unsigned cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    unsigned n = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MACAQ_OK : cuda_fail(e);
}

// ------------------------------------------------------------------------ quantization
template <int kB, bool kWeight, bool kBf16Out = false>
macaq_status run_quant_b(const CUtensorMap &map, const QuantArgs &a, int grid, cudaStream_t st) {
    auto k = quant_kernel<kB, kWeight, kBf16Out>;
    const size_t smem = quant_smem_bytes(a.E);
    macaq_status s = set_smem(k, smem);
    if (s != MACAQ_OK) return s;
    return launch(k, dim3(grid), dim3(kQThreads), smem, st, 1, map, a);
}

template <bool kWeight, bool kBf16Out = false>
macaq_status run_quant(int32_t b, const CUtensorMap &map, const QuantArgs &a, int grid, cudaStream_t st) {
    switch (b) {
        case 1: return run_quant_b<1, kWeight, kBf16Out>(map, a, grid, st);
        case 16: return run_quant_b<16, kWeight, kBf16Out>(map, a, grid, st);
        case 32: return run_quant_b<32, kWeight, kBf16Out>(map, a, grid, st);
        case 64: return run_quant_b<64, kWeight, kBf16Out>(map, a, grid, st);
        case 128: return run_quant_b<128, kWeight, kBf16Out>(map, a, grid, st);
        default: return MACAQ_ERR_UNSUPPORTED;
    }
}

template <int kB>
macaq_status run_quant_gather_b(const QuantArgs &a, const GatherArgs &gx, int grid, cudaStream_t st) {
    auto k = quant_gather_kernel<kB>;
    const size_t smem = 2 * sizeof(int32_t) * (a.E + 1);
    macaq_status s = set_smem(k, smem);
    if (s != MACAQ_OK) return s;
    return launch(k, dim3(grid), dim3(kQConsumers), smem, st, 1, a, gx);
}

macaq_status run_quant_gather(int32_t b, const QuantArgs &a, const GatherArgs &gx, int grid, cudaStream_t st) {
    switch (b) {
        case 1: return run_quant_gather_b<1>(a, gx, grid, st);
        case 16: return run_quant_gather_b<16>(a, gx, grid, st);
        case 32: return run_quant_gather_b<32>(a, gx, grid, st);
        case 64: return run_quant_gather_b<64>(a, gx, grid, st);
        case 128: return run_quant_gather_b<128>(a, gx, grid, st);
        default: return MACAQ_ERR_UNSUPPORTED;
    }
}

// row_index != nullptr: the gather form (activations only): output row m quantizes X row
// row_index[m] of x_rows rows.
// bf16_out: the transform without MXFP4 (activations only): q receives bf16 [rows, K], sf is unused.
macaq_status quantize(const void *X, const float *mul, int64_t rows, int64_t K, int32_t b, bool weight,
                      const int32_t *offsets, int32_t E, uint8_t *q, uint8_t *sf, float *inv_s, cudaStream_t st,
                      const int32_t *row_index = nullptr, int64_t x_rows = 0, bool bf16_out = false) {
    if (rows < 0 || K <= 0 || K % 128 != 0) return MACAQ_ERR_SHAPE;
    if (!valid_block(b)) return MACAQ_ERR_UNSUPPORTED;
    if (offsets != nullptr && (E < 1 || E > 16384)) return MACAQ_ERR_SHAPE;
    if (rows * (K / 32) >= (int64_t(1) << 31)) return MACAQ_ERR_SHAPE;
    if (row_index != nullptr && (x_rows < 1 || x_rows * K >= (int64_t(1) << 40))) return MACAQ_ERR_SHAPE;
    if (rows == 0 && (inv_s == nullptr || mul == nullptr)) return MACAQ_OK;
    if (rows > 0 && (X == nullptr || q == nullptr || (sf == nullptr && !bf16_out))) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(q) || !aligned16(sf) || !aligned16(mul) || !aligned16(inv_s) ||
        !aligned16(offsets) || !aligned16(row_index))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;

    QuantArgs a;
    a.mul = mul;
    a.offsets = offsets;
    a.q = q;
    a.sf = sf;
    a.inv_s = inv_s;
    a.rows = rows;
    a.K = static_cast<uint32_t>(K);
    a.kg = static_cast<uint32_t>(K / 32);
    a.slab_groups = a.kg % 32 == 0 ? 32 : a.kg % 16 == 0 ? 16 : a.kg % 8 == 0 ? 8 : 4;
    a.slab_shift = a.slab_groups == 32 ? 5 : a.slab_groups == 16 ? 4 : a.slab_groups == 8 ? 3 : 2;
    a.slabs = a.kg / a.slab_groups;
    a.tile_rows = kQConsumers / a.slab_groups;
    a.row_tiles = static_cast<uint32_t>((rows + a.tile_rows - 1) / a.tile_rows);
    a.E = offsets ? E : 1;
    a.wait_limit_ns = g_wait_limit_ns.load();

    // CTAs: a multiple of the slab count, at most two per SM, no more than there are row tiles
    uint32_t per_slab = (2u * dev.sms) / a.slabs;
    if (per_slab > a.row_tiles) per_slab = a.row_tiles;
    if (per_slab < 1) per_slab = 1;
    const int grid = static_cast<int>(per_slab * a.slabs);
    if (row_index != nullptr) {
        GatherArgs gx;
        gx.x = static_cast<const uint16_t *>(X);
        gx.row_index = row_index;
        gx.x_rows = x_rows;
        return run_quant_gather(b, a, gx, grid, st);
    }
    CUtensorMap map;
    std::memset(&map, 0, sizeof map);
    if (rows > 0) {
        // X as [rows][K/64 chunks of 128 bytes][64 elements]; a tile is tile_rows x slab x 64
        const uint64_t dims[3] = {64, static_cast<uint64_t>(K) / 64, static_cast<uint64_t>(rows)};
        const uint64_t strides[2] = {128, static_cast<uint64_t>(K) * 2};
        const uint32_t box[3] = {64, a.slab_groups / 2, a.tile_rows};
        s = tensor_map(&map, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (s != MACAQ_OK) return s;
    }
    if (bf16_out) return run_quant<false, true>(b, map, a, grid, st);
    return weight ? run_quant<true>(b, map, a, grid, st) : run_quant<false>(b, map, a, grid, st);
}

// ------------------------------------------------------------------------ GEMM
template <int BN, bool kGrouped>
macaq_status run_gemm(const CUtensorMap &amap, const CUtensorMap &bmap, const GemmArgs &g, dim3 grid,
                      cudaStream_t st) {
    auto k = gemm_mxf4_kernel<BN, kGrouped>;
    const size_t smem = gemm_smem_bytes<BN>(kGrouped ? g.E : 0);
    macaq_status s = set_smem(k, smem);
    if (s != MACAQ_OK) return s;
    return launch(k, grid, dim3(kGemmThreads), smem, st, 1, amap, bmap, g);
}

// ------------------------------------------------------------------------ skinny GEMM (M <= 128)
constexpr int kSkinnyMaxM = 128;
// Workspace layout: per-tile arrival counters in the first 64 KiB (zero between calls; the kernel
// resets every counter it used), then scratch that needs no initial value: the skinny kernel's fp32
// partial tiles, and in the fused two-kernel path the quantized activations after them.
constexpr size_t kCountRegion = 65536;

struct SkinnyPlan {
    bool ok;                   // the tiles' counters fit the counter region
    int32_t mp, stages, max_pieces;
    uint32_t units, gran, ctas, tiles;
    size_t partial_bytes, count_bytes;
};

// Work split of the skinny GEMM on a device with `sms` SMs: equal contiguous ranges of (weight tile,
// K-block) units per CTA, cut either on tile boundaries (every CTA writes whole tiles) or anywhere
// (a tile's pieces meet in the workspace and the CTA that finishes its last piece adds them). The
// plan takes the cheapest of: whole tiles, and splits into at most 2, 3 or 4 pieces per tile on up
// to all SMs, under a time model of the launch: streaming (the larger of the HBM time of all bytes
// and one CTA's bytes at the rate a single SM sustains) plus, for splits, the final reduction (a
// fence and atomic, then one L2 round trip per 16 rows, four pieces at a time).
constexpr int kSkinnyMaxPiecesPerTile = 4;
constexpr double kHbmBytesPerS = 6.0e12;      // sustained HBM read rate of a whole-GPU stream
constexpr double kSmBytesPerS = 40.0e9;       // what one SM's TMA ring sustains on its own
constexpr double kL2RoundTripS = 0.7e-6;      // one dependent L2 load round (reduction)
constexpr double kReduceFixedS = 1.0e-6;      // fence + atomic + barrier before the reduction

SkinnyPlan skinny_plan(int64_t M, int64_t N, int64_t K, int sms, bool fused = false) {
    SkinnyPlan p{};
    p.mp = static_cast<int32_t>((M + 15) / 16 * 16);
    p.tiles = static_cast<uint32_t>(N / 128);
    const uint32_t num_kb = static_cast<uint32_t>(K / 256);
    p.units = p.tiles * num_kb;
    const double w_bytes = static_cast<double>(N) * K * 0.53125;
    const double tile_bytes = w_bytes / p.tiles;
    // pieces of the tile cut most often when `ctas` equal ranges of unit granularity `gran` are used
    auto pieces_of = [&](uint32_t ctas, uint32_t gran) {
        const uint32_t chunks = p.units / gran;
        int mx = 1;
        for (uint32_t t = 0; t < p.tiles; ++t) {
            const uint64_t u0 = static_cast<uint64_t>(t) * num_kb, u1 = u0 + num_kb - 1;
            const uint64_t c0 = ((u0 / gran + 1) * ctas - 1) / chunks, c1 = ((u1 / gran + 1) * ctas - 1) / chunks;
            mx = std::max(mx, static_cast<int>(c1 - c0 + 1));
        }
        return mx;
    };
    // whole tiles
    const uint32_t whole_ctas = std::min<uint32_t>(p.tiles, static_cast<uint32_t>(sms));
    const double whole_per_cta = tile_bytes * ((p.tiles + whole_ctas - 1) / whole_ctas);
    double best = std::max(w_bytes / kHbmBytesPerS, whole_per_cta / kSmBytesPerS);
    p.gran = num_kb;
    p.ctas = whole_ctas;
    p.max_pieces = 1;
    const uint64_t most = std::min<uint64_t>(static_cast<uint64_t>(sms), p.units);
    const uint64_t cands[3] = {std::min<uint64_t>(most, 2ull * p.tiles), std::min<uint64_t>(most, 3ull * p.tiles), most};
    for (uint64_t c : cands) {
        const uint32_t ctas = static_cast<uint32_t>(c);
        if (ctas <= whole_ctas) continue;
        const int pieces = pieces_of(ctas, 1);
        if (pieces > kSkinnyMaxPiecesPerTile) continue;
        const double part_bytes = 2.0 * pieces * p.tiles * M * 128 * 4;
        const double t = std::max((w_bytes + part_bytes) / kHbmBytesPerS, w_bytes / ctas / kSmBytesPerS) +
                         kReduceFixedS + ((M + 15) / 16) * ((pieces + 3) / 4) * kL2RoundTripS;
        if (t < best) {
            best = t;
            p.gran = 1;
            p.ctas = ctas;
            p.max_pieces = pieces;
        }
    }
    const bool split = p.gran == 1;
    p.partial_bytes = split ? static_cast<size_t>(p.tiles) * p.max_pieces * static_cast<size_t>(M) * 128 * 4 : 0;
    p.count_bytes = kCountRegion;
    p.ok = static_cast<size_t>(p.tiles) * 4 <= kCountRegion;
    const int smem_budget = 232448 - 1024 - 1024 - skinny_stage_bytes_y(p.mp);  // minus slack, static data, Y staging
    int st = smem_budget / (fused ? skinny_stage_bytes_fused(p.mp) : skinny_stage_bytes(p.mp));
    p.stages = st > kSkinnyMaxStages ? kSkinnyMaxStages : st;
    return p;
}

// skinny_plan() memoised per (shape, SM count, form): it runs on every call.
SkinnyPlan skinny_plan_cached(int64_t M, int64_t N, int64_t K, int sms, bool fused = false) {
    static std::mutex mu;
    static std::map<std::tuple<int64_t, int64_t, int64_t, int, bool>, SkinnyPlan> cache;
    const auto key = std::make_tuple(M, N, K, sms, fused);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    const SkinnyPlan p = skinny_plan(M, N, K, sms, fused);
    if (cache.size() > 4096) cache.clear();
    cache.emplace(key, p);
    return p;
}

// The skinny GEMM. fused_b = 0: A is Xq/Asf (quantized activations). fused_b > 0: A is bf16 X
// (M <= kSkinnyFusedMaxM) and the kernel applies 1/s (inv_s, may be null), H_b and MXFP4 itself.
template <int kFusedB>
macaq_status launch_skinny(const CUtensorMap &wmap, const CUtensorMap &xmap, const CUtensorMap &sfwmap,
                           const CUtensorMap &sfxmap, const CUtensorMap &ymap, const SkinnyArgs &g, const SkinnyPlan &p,
                           cudaStream_t st) {
    const int sb = kFusedB > 0 ? skinny_stage_bytes_fused(p.mp) : skinny_stage_bytes(p.mp);
    const size_t smem = 1024 + static_cast<size_t>(p.stages) * sb + skinny_stage_bytes_y(p.mp);
    macaq_status s = set_smem(gemm_mxf4_skinny_kernel<kFusedB>, smem);
    if (s != MACAQ_OK) return s;
    return launch(gemm_mxf4_skinny_kernel<kFusedB>, dim3(p.ctas), dim3(kFusedB > 0 ? 320 : 192), smem, st, 1, wmap, xmap,
                  sfwmap, sfxmap, ymap, g);
}

// clear_counts > 0: zero that many bytes at the start of the workspace on `st` right before the
// launch, once every argument and descriptor has been accepted (the fixed-scratch entry point).
macaq_status run_skinny(const void *A, const uint8_t *Asf, const float *inv_s, int32_t fused_b, int64_t M, int64_t N,
                        int64_t K, const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype, void *workspace,
                        size_t ws_bytes, int sms, cudaStream_t st, size_t clear_counts = 0) {
    const bool fused = fused_b > 0;
    const SkinnyPlan p = skinny_plan_cached(M, N, K, sms, fused);
    if (!p.ok) return MACAQ_ERR_SHAPE;
    // the in-kernel quantizer warps take the stages in turn, four at a time: a stage count that is
    // not a multiple of four would give one stage to two warps at different phases
    if (fused && p.stages % 4 != 0) return MACAQ_ERR_UNSUPPORTED;
    if (fused && M > kSkinnyFusedMaxM) return MACAQ_ERR_SHAPE;   // the only sizes it is tested for
    if (ws_bytes < p.partial_bytes + p.count_bytes) return MACAQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MACAQ_ERR_ALIGNMENT;
    CUtensorMap wmap, xmap, sfwmap, sfxmap, ymap;
    macaq_status s = tensor_map_2d(&wmap, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, kBKBytes, 128,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (s == MACAQ_OK) {
        if (fused)  // bf16 X, one K-block (256 elements) of all 16 rows per box; rows past M read as zero
            s = tensor_map_2d(&xmap, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 256, p.mp,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
        else
            s = tensor_map_2d(&xmap, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, M, K / 2, kBKBytes, p.mp,
                              CU_TENSOR_MAP_SWIZZLE_128B);
    }
    // replicated scale factors: (128 B, the K-block's two tiles, 8-row group, replica (stride 0), tile)
    const uint32_t sbox[5] = {128, 2, 4, 4, 1};
    const uint64_t sstr[4] = {512, 128, 0, 512};
    if (s == MACAQ_OK) {
        const uint64_t d[5] = {128, 2, 4, 4, macaq_sf_bytes(N, K) / 512};
        s = tensor_map(&sfwmap, Wsf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, d, sstr, sbox, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (s == MACAQ_OK) {
        if (fused) {
            sfxmap = sfwmap;  // unused: the kernel writes X's scale factors itself
        } else {
            const uint64_t d[5] = {128, 2, 4, 4, macaq_sf_bytes(M, K) / 512};
            s = tensor_map(&sfxmap, Asf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, d, sstr, sbox, CU_TENSOR_MAP_SWIZZLE_NONE);
        }
    }
    // Y as bf16 [M, N]; each epilogue warp stores a 32-column x Mp-row box
    if (s == MACAQ_OK)
        s = tensor_map_2d(&ymap, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 32, p.mp, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (s != MACAQ_OK) return s;
    SkinnyArgs g;
    g.y = Y;
    g.counts = static_cast<int32_t *>(workspace);
    g.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + p.count_bytes);
    g.M = static_cast<int32_t>(M);
    g.N = static_cast<int32_t>(N);
    g.K = static_cast<int32_t>(K);
    g.mp = p.mp;
    g.out_f32 = out_dtype == MACAQ_OUT_F32;
    g.stages = p.stages;
    g.max_pieces = p.max_pieces;
    g.units = p.units;
    g.gran = p.gran;
    g.wait_limit_ns = g_wait_limit_ns.load();
    g.inv_s = inv_s;
    if (clear_counts > 0) {
        const cudaError_t e = cudaMemsetAsync(workspace, 0, clear_counts, st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    switch (fused_b) {
        case 0: return launch_skinny<0>(wmap, xmap, sfwmap, sfxmap, ymap, g, p, st);
        case 1: return launch_skinny<1>(wmap, xmap, sfwmap, sfxmap, ymap, g, p, st);
        case 16: return launch_skinny<16>(wmap, xmap, sfwmap, sfxmap, ymap, g, p, st);
        case 32: return launch_skinny<32>(wmap, xmap, sfwmap, sfxmap, ymap, g, p, st);
        case 64: return launch_skinny<64>(wmap, xmap, sfwmap, sfxmap, ymap, g, p, st);
        case 128: return launch_skinny<128>(wmap, xmap, sfwmap, sfxmap, ymap, g, p, st);
        default: return MACAQ_ERR_UNSUPPORTED;
    }
}

// The dense GEMM on 2-SM pairs (M > 128, N % 256 == 0, K % 256 == 0). swiglu_b > 0 selects the fused
// SwiGLU epilogue (the down projection's quantized input goes to `so` instead of Y).
template <int kSwiglu, int kFusedB = 0>
macaq_status launch_pair(const CUtensorMap &amap, const CUtensorMap &bmap, const CUtensorMap &sfamap,
                         const CUtensorMap &sfbmap, const CUtensorMap &ymap, const GemmArgs &g, int replica_boxes,
                         const SwigluOut &so, const FusedA &fa, unsigned pairs, cudaStream_t st) {
    constexpr bool kGrouped = kSwiglu < 0;   // kSwiglu = -1 selects the grouped form
    auto k = gemm_mxf4_pair_kernel<kGrouped ? 0 : kSwiglu, kFusedB, kGrouped>;
    // the grouped form keeps three [E + 1] arrays of the expert layout after the epilogue buffers
    const size_t smem = PairCfg::kSmemBytes + (kGrouped ? 3 * sizeof(int32_t) * (g.E + 1) : 0);
    macaq_status s = set_smem(k, smem);
    if (s != MACAQ_OK) return s;
    return launch(k, dim3(2 * pairs), dim3(PairCfg::kThreads), smem, st, 2, amap, bmap, sfamap, sfbmap, ymap, g,
                  replica_boxes, so, fa);
}

// fused_b > 0: A and Asf are the workspace buffers that the kernel itself fills from fa.x (the fused
// layer's in-kernel quantization with Hadamard block fused_b).
macaq_status run_pair(const uint8_t *A, const uint8_t *Asf, int64_t rows, int64_t N, int64_t K, const uint8_t *Wq,
                      const uint8_t *Wsf, void *Y, int32_t out_dtype, const GemmArgs &g, int32_t swiglu_b,
                      const SwigluOut &so, int sms, cudaStream_t st, int32_t fused_b = 0, const FusedA &fa = FusedA{}) {
    macaq_status s;
    // grouped form (g.offsets set): W is E stacked [N, K/2] blocks with their SF one after another,
    // and A's SF starts each expert on a fresh 128-row tile
    const bool grouped = g.offsets != nullptr;
    const int64_t experts = grouped ? g.E : 1;
    const uint64_t sfa_bytes = grouped ? macaq_grouped_sf_bytes(rows, g.E, K) : macaq_sf_bytes(rows, K);
    const uint64_t sfb_bytes = static_cast<uint64_t>(experts) * macaq_sf_bytes(N, K);
    CUtensorMap amap, bmap, sfamap, sfbmap;
    s = tensor_map_2d(&amap, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, rows, K / 2, kBKBytes, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (s == MACAQ_OK)
        s = tensor_map_2d(&bmap, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, experts * N, K / 2, kBKBytes, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    // replica views of the SF buffers: (128 B, half h, 8-row group i, 128x4 tile c); for A the
    // halves are the K-block's two tiles (512 B apart), for B the two 128-row tiles of the
    // 256-row N tile (K/128 tiles apart)
    const uint64_t kq = static_cast<uint64_t>(K / 128);
    // one 4 KB box holding all four replicas needs a zero-stride replica dimension; if the driver
    // refuses that view, four 1 KB boxes (one replica each) are used instead
    int replica_boxes = 1;
    if (s == MACAQ_OK) {
        const uint64_t da[5] = {128, 2, 4, 4, sfa_bytes / 512};
        const uint64_t sa[4] = {512, 128, 0, 512};
        const uint64_t db[5] = {128, 2, 4, 4, sfb_bytes / 512};
        const uint64_t sb[4] = {kq * 512, 128, 0, 512};
        const uint32_t box[5] = {128, 2, 4, 4, 1};
        if (tensor_map(&sfamap, Asf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, da, sa, box, CU_TENSOR_MAP_SWIZZLE_NONE) != MACAQ_OK ||
            tensor_map(&sfbmap, Wsf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, db, sb, box, CU_TENSOR_MAP_SWIZZLE_NONE) != MACAQ_OK) {
            replica_boxes = 4;
            const uint64_t da4[4] = {128, 2, 4, sfa_bytes / 512};
            const uint64_t sa4[3] = {512, 128, 512};
            const uint64_t db4[4] = {128, 2, 4, sfb_bytes / 512};
            const uint64_t sb4[3] = {kq * 512, 128, 512};
            const uint32_t box4[4] = {128, 2, 4, 1};
            s = tensor_map(&sfamap, Asf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, da4, sa4, box4, CU_TENSOR_MAP_SWIZZLE_NONE);
            if (s == MACAQ_OK)
                s = tensor_map(&sfbmap, Wsf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, db4, sb4, box4, CU_TENSOR_MAP_SWIZZLE_NONE);
        }
    }
    // Y in 32-row x 128-byte boxes, 128-byte swizzled (the epilogue's staging layout)
    CUtensorMap ymap = amap;   // the fused SwiGLU epilogue writes no Y (the map is not used)
    if (s == MACAQ_OK && swiglu_b == 0) {
        const bool f32 = out_dtype == MACAQ_OUT_F32;
        s = tensor_map_2d(&ymap, Y, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, rows,
                          N * (f32 ? 4 : 2), f32 ? 32 : 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (s != MACAQ_OK) return s;
    // grouped: the tile count is known on the device only; sum ceil(tiles_e / 2) <= rows / 256 + E
    const int64_t tiles = ((rows + 255) / 256 + (grouped ? experts : 0)) * (N / 256);
    const int64_t max_pairs = sms / 2;
    const unsigned pairs = static_cast<unsigned>(tiles < max_pairs ? tiles : max_pairs);
    if (grouped) return launch_pair<-1>(amap, bmap, sfamap, sfbmap, ymap, g, replica_boxes, so, fa, pairs, st);
    if (fused_b > 0) {
        // in-GEMM quantization: raster bands of about two rounds of tiles, so the first round needs
        // only the first band's rows of A; the units follow the same bands
        const int64_t n_tiles = N / 256;
        const int64_t band = std::min<int64_t>(kRasterM, std::max<int64_t>(2, (2 * pairs + n_tiles - 1) / n_tiles));
        GemmArgs gb = g;
        gb.raster_m = static_cast<int32_t>(band);
        FusedA fb = fa;
        fb.band_rt = static_cast<int32_t>(2 * band);
        switch (fused_b) {
            case 1: return launch_pair<0, 1>(amap, bmap, sfamap, sfbmap, ymap, gb, replica_boxes, so, fb, pairs, st);
            case 16: return launch_pair<0, 16>(amap, bmap, sfamap, sfbmap, ymap, gb, replica_boxes, so, fb, pairs, st);
            case 32: return launch_pair<0, 32>(amap, bmap, sfamap, sfbmap, ymap, gb, replica_boxes, so, fb, pairs, st);
            case 64: return launch_pair<0, 64>(amap, bmap, sfamap, sfbmap, ymap, gb, replica_boxes, so, fb, pairs, st);
            case 128: return launch_pair<0, 128>(amap, bmap, sfamap, sfbmap, ymap, gb, replica_boxes, so, fb, pairs, st);
            default: return MACAQ_ERR_UNSUPPORTED;
        }
    }
    switch (swiglu_b) {
        case 0: return launch_pair<0>(amap, bmap, sfamap, sfbmap, ymap, g, replica_boxes, so, fa, pairs, st);
        case 1: return launch_pair<1>(amap, bmap, sfamap, sfbmap, ymap, g, replica_boxes, so, fa, pairs, st);
        case 16: return launch_pair<16>(amap, bmap, sfamap, sfbmap, ymap, g, replica_boxes, so, fa, pairs, st);
        case 32: return launch_pair<32>(amap, bmap, sfamap, sfbmap, ymap, g, replica_boxes, so, fa, pairs, st);
        case 64: return launch_pair<64>(amap, bmap, sfamap, sfbmap, ymap, g, replica_boxes, so, fa, pairs, st);
        default: return MACAQ_ERR_UNSUPPORTED;
    }
}

macaq_status gemm(const uint8_t *A, const uint8_t *Asf, const int32_t *offsets, int32_t E, int64_t rows, int64_t N,
                  int64_t K, const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype, void *workspace,
                  size_t ws_bytes, cudaStream_t st) {
    if (rows < 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 128 != 0) return MACAQ_ERR_SHAPE;
    if (rows >= (int64_t(1) << 31) || static_cast<int64_t>(E) * N >= (int64_t(1) << 31)) return MACAQ_ERR_SHAPE;
    if (out_dtype != MACAQ_OUT_BF16 && out_dtype != MACAQ_OUT_F32) return MACAQ_ERR_INVALID_ARG;
    if (offsets != nullptr && (E < 1 || E > 1024)) return MACAQ_ERR_SHAPE;
    if (rows == 0) return MACAQ_OK;
    if (A == nullptr || Asf == nullptr || Wq == nullptr || Wsf == nullptr || Y == nullptr)
        return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(Asf) || !aligned16(Wq) || !aligned16(Wsf) || !aligned16(Y) ||
        !aligned16(offsets))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;

    if (offsets == nullptr && rows <= kSkinnyMaxM && K % 256 == 0 && workspace != nullptr &&
        skinny_plan_cached(rows, N, K, dev.sms).ok)
        return run_skinny(A, Asf, nullptr, 0, rows, N, K, Wq, Wsf, Y, out_dtype, workspace, ws_bytes, dev.sms, st);

    const int BN = (N % 256 == 0) ? 256 : 128;
    const bool grouped = offsets != nullptr;
    // 2-SM pairs, 256 x 256 tiles: dense calls with more than 128 rows, grouped calls whose experts
    // average at least 256 rows (fewer rows per expert leave too many half-empty pairs)
    const bool pair = BN == 256 && K % 256 == 0 &&
                      (grouped ? (E <= 1024 && rows >= 256 * static_cast<int64_t>(E)) : rows > 128);
    const int32_t experts = grouped ? E : 1;
    GemmArgs g{};
    g.asf = Asf;
    g.bsf = Wsf;
    g.y = Y;
    g.offsets = offsets;
    g.rows = rows;
    g.N = static_cast<int32_t>(N);
    g.K = static_cast<int32_t>(K);
    g.E = experts;
    g.out_f32 = out_dtype == MACAQ_OUT_F32;
    g.bsf_stride = macaq_sf_bytes(N, K);
    g.wait_limit_ns = g_wait_limit_ns.load();

    if (pair) return run_pair(A, Asf, rows, N, K, Wq, Wsf, Y, out_dtype, g, 0, SwigluOut{}, dev.sms, st);

    CUtensorMap amap, bmap;
    s = tensor_map_2d(&amap, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, rows, K / 2, kBKBytes, kBM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MACAQ_OK) return s;
    s = tensor_map_2d(&bmap, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, static_cast<uint64_t>(experts) * N, K / 2,
                      kBKBytes, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MACAQ_OK) return s;

    // persistent: at most one CTA per SM; the CTAs walk the tiles (grouped: the tile count is
    // only known on the device, so the bound uses ceil(rows/128) + E row tiles)
    const int64_t m_tiles = grouped ? (rows + 127) / 128 + experts : (rows + 127) / 128;
    const int64_t tiles = m_tiles * (N / BN);
    const unsigned grid = static_cast<unsigned>(tiles < dev.sms ? tiles : dev.sms);
    if (BN == 256) return grouped ? run_gemm<256, true>(amap, bmap, g, dim3(grid), st) : run_gemm<256, false>(amap, bmap, g, dim3(grid), st);
    return grouped ? run_gemm<128, true>(amap, bmap, g, grid, st) : run_gemm<128, false>(amap, bmap, g, grid, st);
}

}  // namespace
// ------------------------------------------------------------------------ fixed scratch
// Scratch of the skinny kernel for callers that may not allocate device memory: it is part of the
// module's static device data, so it exists as soon as the module is loaded on a device.
__device__ __align__(256) uint8_t g_fixed_scratch[MACAQ_FIXED_SCRATCH_BYTES];

// Device address of g_fixed_scratch on the current device. In host code the symbol is only a
// host-side stand-in, so the address is looked up on every call (a host-side table lookup once the
// module is loaded); nothing is cached, so a device reset that reloads the module is harmless.
macaq_status fixed_scratch(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fixed_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    *out = p;
    return MACAQ_OK;
}

macaq_status linear_fixed_scratch(const uint8_t *A, const uint8_t *Asf, int64_t M, int64_t N, int64_t K,
                                  const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype,
                                  cudaStream_t st) {
    const bool skinny = M >= 1 && M <= kSkinnyMaxM && N > 0 && N % 128 == 0 && K > 0 && K % 256 == 0 &&
                        N < (int64_t(1) << 31) && K < (int64_t(1) << 31);
    if (!skinny) return gemm(A, Asf, nullptr, 1, M, N, K, Wq, Wsf, Y, out_dtype, nullptr, 0, st);
    // every check of the skinny path comes before the counter clear, so a refused call enqueues nothing
    if (out_dtype != MACAQ_OUT_BF16 && out_dtype != MACAQ_OUT_F32) return MACAQ_ERR_INVALID_ARG;
    if (A == nullptr || Asf == nullptr || Wq == nullptr || Wsf == nullptr || Y == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(Asf) || !aligned16(Wq) || !aligned16(Wsf) || !aligned16(Y))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;
    const SkinnyPlan p = skinny_plan_cached(M, N, K, dev.sms);
    if (!p.ok) return gemm(A, Asf, nullptr, 1, M, N, K, Wq, Wsf, Y, out_dtype, nullptr, 0, st);
    if (p.partial_bytes + p.count_bytes > MACAQ_FIXED_SCRATCH_BYTES) return MACAQ_ERR_WORKSPACE;
    void *scratch = nullptr;
    s = fixed_scratch(&scratch);
    if (s != MACAQ_OK) return s;
    // only the per-tile counters this call uses must start at zero; run_skinny clears them on `st`
    // after its descriptors are built, immediately before the launch
    const size_t used_counts = (static_cast<size_t>(p.tiles) * 4 + 255) / 256 * 256;
    return run_skinny(A, Asf, nullptr, 0, M, N, K, Wq, Wsf, Y, out_dtype, scratch, MACAQ_FIXED_SCRATCH_BYTES, dev.sms,
                      st, used_counts);
}

// ------------------------------------------------------------------------ fused layer (a7)
// Workspace of the fused layer: the GEMM's own region (skinny counters and partials, when the skinny
// kernel runs), then room for the quantized activations and their scale factors, which the two-kernel
// form writes and reads back. Offsets are 256-byte aligned.
struct FusedLayout {
    size_t gemm_ws;   // the skinny kernel's region (counters + partials), 0 when it does not run
    size_t a_off, sf_off, total;
    bool in_kernel;   // the skinny kernel quantizes X itself
    bool in_pair;     // the 2-SM GEMM quantizes X itself (one launch; ready counts in the counter region)
};

FusedLayout fused_layout(int64_t M, int64_t N, int64_t K, int32_t E, int sms) {
    FusedLayout f{};
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    if (E == 0 && M >= 1 && M <= kSkinnyMaxM && K % 256 == 0) {
        const SkinnyPlan p = skinny_plan_cached(M, N, K, sms, M <= kSkinnyFusedMaxM);
        if (p.ok) {
            f.gemm_ws = up(p.count_bytes + p.partial_bytes);
            // the quantizer warps need a stage count that is a multiple of four (run_skinny checks it)
            f.in_kernel = M <= kSkinnyFusedMaxM && p.stages % 4 == 0;
        }
    }
    // large M on 2-SM pairs: the ready counts, the work counter and the exit counter fit the region
    f.in_pair = E == 0 && M > kSkinnyMaxM && N % 256 == 0 && K % 256 == 0 &&
                static_cast<size_t>((M + 127) / 128) * (K / 256 + 1) + 2 <= kCountRegion / 4;
    // the activations never overlap the counter region, whichever kernel runs afterwards
    f.a_off = std::max(f.gemm_ws, up(kCountRegion));
    f.sf_off = f.a_off + up(static_cast<size_t>(M) * static_cast<size_t>(K / 2));
    f.total = f.sf_off + (E > 0 ? macaq_grouped_sf_bytes(M, E, K) : macaq_sf_bytes(M, K));
    return f;
}

// Y = (X diag(1/s) H_b, MXFP4) x W'^T from bf16 X. Dense calls with M <= 4 and K % 256 == 0 run the
// skinny kernel with its quantizer warps: no quantized activation touches HBM. Every other shape (and
// every grouped call) quantizes X into the workspace and runs the GEMM on it, two launches in stream
// order: re-quantizing an A tile for every output tile it meets would cost more than the
// 0.53125 B/element round trip once M is large. one_launch: dense M > 128 with N, K % 256 == 0 runs
// the 2-SM GEMM that quantizes X itself (one launch, ready counts in the counter region).
macaq_status linear_fused(const void *X, const float *inv_s, int32_t b, const int32_t *offsets, int32_t E, int64_t M,
                          int64_t N, int64_t K, const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype,
                          void *workspace, size_t ws_bytes, cudaStream_t st, bool one_launch = false) {
    if (M < 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 128 != 0) return MACAQ_ERR_SHAPE;
    if (!valid_block(b)) return MACAQ_ERR_UNSUPPORTED;
    if (offsets != nullptr && (E < 1 || E > 1024)) return MACAQ_ERR_SHAPE;
    if (out_dtype != MACAQ_OUT_BF16 && out_dtype != MACAQ_OUT_F32) return MACAQ_ERR_INVALID_ARG;
    if (M == 0) return MACAQ_OK;
    if (X == nullptr || Wq == nullptr || Wsf == nullptr || Y == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(inv_s) || !aligned16(Wq) || !aligned16(Wsf) || !aligned16(Y) ||
        !aligned16(workspace) || !aligned16(offsets))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;
    const FusedLayout f = fused_layout(M, N, K, offsets != nullptr ? E : 0, dev.sms);
    if (workspace == nullptr || ws_bytes < f.total) return MACAQ_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (offsets == nullptr && f.in_kernel)
        return run_skinny(X, nullptr, inv_s, b, M, N, K, Wq, Wsf, Y, out_dtype, ws, f.gemm_ws, dev.sms, st);
    if (one_launch && offsets == nullptr && f.in_pair) {
        // one launch: the 2-SM GEMM quantizes X into the workspace itself (ready counts in the
        // counter region) and reads A from there
        FusedA fa{};
        fa.x = static_cast<const uint16_t *>(X);
        fa.inv_s = inv_s;
        fa.xq = ws + f.a_off;
        fa.xsf = ws + f.sf_off;
        fa.rt_count = static_cast<int32_t>((M + 127) / 128);
        fa.kb_count = static_cast<int32_t>(K / 256);
        fa.units = fa.rt_count * fa.kb_count * kFaUnitsPerBlock;
        int32_t *counters = reinterpret_cast<int32_t *>(ws);
        fa.flags = counters;
        fa.rt_done = counters + fa.rt_count * fa.kb_count;
        fa.next_unit = fa.rt_done + fa.rt_count;
        fa.exit_count = fa.next_unit + 1;
        GemmArgs g{};
        g.asf = ws + f.sf_off;
        g.bsf = Wsf;
        g.y = Y;
        g.offsets = nullptr;
        g.rows = M;
        g.N = static_cast<int32_t>(N);
        g.K = static_cast<int32_t>(K);
        g.E = 1;
        g.out_f32 = out_dtype == MACAQ_OUT_F32;
        g.bsf_stride = macaq_sf_bytes(N, K);
        g.wait_limit_ns = g_wait_limit_ns.load();
        return run_pair(ws + f.a_off, ws + f.sf_off, M, N, K, Wq, Wsf, Y, out_dtype, g, 0, SwigluOut{}, dev.sms, st, b, fa);
    }
    s = quantize(X, inv_s, M, K, b, false, offsets, offsets != nullptr ? E : 0, ws + f.a_off, ws + f.sf_off, nullptr, st);
    if (s != MACAQ_OK) return s;
    return gemm(ws + f.a_off, ws + f.sf_off, offsets, offsets != nullptr ? E : 1, M, N, K, Wq, Wsf, Y, out_dtype,
                f.gemm_ws > 0 ? ws : nullptr, f.gemm_ws, st);
}

// ------------------------------------------------------------------------ weight-only (W4A16)
struct WonlyLayout {
    bool ok;
    SkinnyPlan plan;
    int32_t stages;
    size_t gemm_ws, xt_off, total;
};

WonlyLayout wonly_layout(int64_t M, int64_t N, int64_t K, int sms) {
    WonlyLayout l{};
    if (M < 1 || M > kWoMaxM || N <= 0 || N % 128 != 0 || K <= 0 || K % 256 != 0) return l;
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    l.plan = skinny_plan_cached(M, N, K, sms);
    const int budget = 232448 - 1024 - 1024 - kWoTableBytes - skinny_stage_bytes_y(l.plan.mp);
    l.stages = std::min(kWoMaxStages, budget / wo_stage_bytes(l.plan.mp));
    l.ok = l.plan.ok && l.stages >= 2;
    l.gemm_ws = up(l.plan.count_bytes + l.plan.partial_bytes);
    l.xt_off = l.gemm_ws;
    l.total = l.xt_off + up(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
    return l;
}

macaq_status act_transform(const void *X, const float *inv_s, int64_t M, int64_t K, int32_t b, void *Xt, cudaStream_t st) {
    return quantize(X, inv_s, M, K, b, false, nullptr, 0, static_cast<uint8_t *>(Xt), nullptr, nullptr, st, nullptr, 0,
                    true);
}

macaq_status linear_w4a16(const void *X, const float *inv_s, int64_t M, int64_t N, int64_t K, int32_t b,
                          const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype, void *workspace,
                          size_t ws_bytes, cudaStream_t st) {
    if (M < 0 || N <= 0 || N % 128 != 0 || K <= 0 || K % 256 != 0 || M > kWoMaxM || N >= (int64_t(1) << 31))
        return MACAQ_ERR_SHAPE;
    if (!valid_block(b)) return MACAQ_ERR_UNSUPPORTED;
    if (out_dtype != MACAQ_OUT_BF16 && out_dtype != MACAQ_OUT_F32) return MACAQ_ERR_INVALID_ARG;
    if (M == 0) return MACAQ_OK;
    if (X == nullptr || Wq == nullptr || Wsf == nullptr || Y == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(inv_s) || !aligned16(Wq) || !aligned16(Wsf) || !aligned16(Y) || !aligned16(workspace))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;
    const WonlyLayout l = wonly_layout(M, N, K, dev.sms);
    if (!l.ok) return MACAQ_ERR_SHAPE;
    if (workspace == nullptr || ws_bytes < l.total) return MACAQ_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *xt = ws + l.xt_off;
    const SkinnyPlan &p = l.plan;
    CUtensorMap wmap, xmap, ymap;
    s = tensor_map_2d(&wmap, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, kBKBytes, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s == MACAQ_OK)   // X' bf16: 64-column atoms of all mp rows (rows past M read as zero)
        s = tensor_map_2d(&xmap, xt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, p.mp, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s == MACAQ_OK)
        s = tensor_map_2d(&ymap, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 32, p.mp, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (s != MACAQ_OK) return s;
    s = act_transform(X, inv_s, M, K, b, xt, st);
    if (s != MACAQ_OK) return s;
    SkinnyArgs g{};
    g.y = Y;
    g.counts = reinterpret_cast<int32_t *>(ws);
    g.partials = reinterpret_cast<float *>(ws + p.count_bytes);
    g.M = static_cast<int32_t>(M);
    g.N = static_cast<int32_t>(N);
    g.K = static_cast<int32_t>(K);
    g.mp = p.mp;
    g.out_f32 = out_dtype == MACAQ_OUT_F32;
    g.stages = l.stages;
    g.max_pieces = p.max_pieces;
    g.units = p.units;
    g.gran = p.gran;
    g.wait_limit_ns = g_wait_limit_ns.load();
    g.inv_s = nullptr;
    const size_t smem = 1024 + static_cast<size_t>(l.stages) * wo_stage_bytes(p.mp) + kWoTableBytes +
                        skinny_stage_bytes_y(p.mp);
    s = set_smem(gemm_w4a16_skinny_kernel, smem);
    if (s != MACAQ_OK) return s;
    return launch(gemm_w4a16_skinny_kernel, dim3(p.ctas), dim3(kWoThreads), smem, st, 1, wmap, xmap, ymap, g, Wsf);
}

// ------------------------------------------------------------------------ SwiGLU -> down-projection input
bool valid_swiglu_block(int32_t b) { return b == 1 || b == 16 || b == 32 || b == 64; }

template <int kB>
macaq_status launch_swiglu_quant(const float *gu, int64_t M, const SwigluOut &o, int sms, cudaStream_t st) {
    const int64_t items = static_cast<int64_t>(o.rows_sf) * (o.I / 64);
    int64_t blocks = (items + 255) / 256;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    if (blocks > cap) blocks = cap;
    return launch(swiglu_quant_kernel<kB>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, 1, gu, M, o);
}

// H' = MXFP4(swiglu(G, U) diag(inv_s) H_b) from a gate/up output in memory (fp32 [M, 2I], 64-interleaved).
macaq_status swiglu_quant(const float *gu, int64_t M, int64_t I, const float *inv_s, int32_t b, uint8_t *hq, uint8_t *hsf,
                          cudaStream_t st) {
    if (M < 0 || I <= 0 || I % 128 != 0 || M >= (int64_t(1) << 31) || I >= (int64_t(1) << 30)) return MACAQ_ERR_SHAPE;
    if (!valid_swiglu_block(b)) return MACAQ_ERR_UNSUPPORTED;
    if (M == 0) return MACAQ_OK;
    if (gu == nullptr || hq == nullptr || hsf == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(gu) || !aligned16(inv_s) || !aligned16(hq) || !aligned16(hsf)) return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;
    SwigluOut o{inv_s, hq, hsf, static_cast<int32_t>(I), static_cast<int32_t>((M + 127) / 128 * 128)};
    switch (b) {
        case 1: return launch_swiglu_quant<1>(gu, M, o, dev.sms, st);
        case 16: return launch_swiglu_quant<16>(gu, M, o, dev.sms, st);
        case 32: return launch_swiglu_quant<32>(gu, M, o, dev.sms, st);
        default: return launch_swiglu_quant<64>(gu, M, o, dev.sms, st);
    }
}

// Whether the gate/up GEMM of these sizes runs the fused epilogue (2-SM pair kernel), and otherwise
// the workspace of the two-step form: the skinny GEMM's region (when it runs), then the fp32 gate/up
// output.
struct SwigluLayout {
    bool fused;
    size_t gemm_ws, gu_off, total;
};

SwigluLayout swiglu_layout(int64_t M, int64_t N, int64_t K, int sms) {
    SwigluLayout l{};
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    l.fused = M > kSkinnyMaxM && N % 256 == 0 && K % 256 == 0;
    if (l.fused) return l;
    if (M >= 1 && M <= kSkinnyMaxM && K % 256 == 0) {
        const SkinnyPlan p = skinny_plan_cached(M, N, K, sms);
        if (p.ok) l.gemm_ws = up(p.count_bytes + p.partial_bytes);
    }
    l.gu_off = std::max(l.gemm_ws, up(kCountRegion));
    l.total = l.gu_off + up(static_cast<size_t>(M) * static_cast<size_t>(N) * 4);
    return l;
}

macaq_status linear_swiglu(const uint8_t *A, const uint8_t *Asf, int64_t M, int64_t N, int64_t K, const uint8_t *Wq,
                           const uint8_t *Wsf, const float *inv_s, int32_t b, uint8_t *hq, uint8_t *hsf, void *workspace,
                           size_t ws_bytes, cudaStream_t st) {
    if (M < 0 || N <= 0 || N % 256 != 0 || K <= 0 || K % 128 != 0) return MACAQ_ERR_SHAPE;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return MACAQ_ERR_SHAPE;
    if (!valid_swiglu_block(b)) return MACAQ_ERR_UNSUPPORTED;
    if (M == 0) return MACAQ_OK;
    if (A == nullptr || Asf == nullptr || Wq == nullptr || Wsf == nullptr || hq == nullptr || hsf == nullptr)
        return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(Asf) || !aligned16(Wq) || !aligned16(Wsf) || !aligned16(inv_s) || !aligned16(hq) ||
        !aligned16(hsf) || !aligned16(workspace))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;
    const SwigluLayout l = swiglu_layout(M, N, K, dev.sms);
    const int64_t I = N / 2;
    if (l.fused) {
        GemmArgs g{};
        g.asf = Asf;
        g.bsf = Wsf;
        g.y = nullptr;
        g.offsets = nullptr;
        g.rows = M;
        g.N = static_cast<int32_t>(N);
        g.K = static_cast<int32_t>(K);
        g.E = 1;
        g.out_f32 = 0;
        g.bsf_stride = macaq_sf_bytes(N, K);
        g.wait_limit_ns = g_wait_limit_ns.load();
        SwigluOut o{inv_s, hq, hsf, static_cast<int32_t>(I), static_cast<int32_t>((M + 127) / 128 * 128)};
        return run_pair(A, Asf, M, N, K, Wq, Wsf, nullptr, MACAQ_OUT_BF16, g, b, o, dev.sms, st);
    }
    if (workspace == nullptr || ws_bytes < l.total) return MACAQ_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *gu = reinterpret_cast<float *>(ws + l.gu_off);
    s = gemm(A, Asf, nullptr, 1, M, N, K, Wq, Wsf, gu, MACAQ_OUT_F32, l.gemm_ws > 0 ? ws : nullptr, l.gemm_ws, st);
    if (s != MACAQ_OK) return s;
    return swiglu_quant(gu, M, I, inv_s, b, hq, hsf, st);
}

// ------------------------------------------------------------------------ Flip-Refinement
template <int kCols, int kR>
macaq_status launch_flip(const FlipArgs &f, int sms, cudaStream_t st) {
    auto k = flip_refine_kernel<kCols, kR>;
    const size_t smem = flip_smem_bytes(kR, f.K);
    macaq_status s = set_smem(k, smem);
    if (s != MACAQ_OK) return s;
    const int64_t groups = (static_cast<int64_t>(f.N) + kR - 1) / kR;
    const unsigned grid = static_cast<unsigned>(groups < sms ? groups : sms);
    return launch(k, dim3(grid), dim3(kFlipThreads), smem, st, 1, f);
}

macaq_status flip_refine(const void *W, const float *s, int64_t N, int64_t K, int32_t b, const float *H, int32_t sweeps,
                         uint8_t *Wq, const uint8_t *Wsf, int32_t *flips, cudaStream_t st) {
    if (N < 0 || K <= 0 || K % 128 != 0 || K > 16384 || N >= (int64_t(1) << 31) || sweeps < 0) return MACAQ_ERR_SHAPE;
    if (!valid_block(b)) return MACAQ_ERR_UNSUPPORTED;
    if (N == 0 || sweeps == 0) return MACAQ_OK;
    if (W == nullptr || H == nullptr || Wq == nullptr || Wsf == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(s) || !aligned16(H) || !aligned16(Wq) || !aligned16(Wsf) ||
        (reinterpret_cast<uintptr_t>(flips) & 3u))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status st_ = device_info(&dev);
    if (st_ != MACAQ_OK) return st_;
    FlipArgs f;
    f.w = static_cast<const uint16_t *>(W);
    f.s = s;
    f.h = H;
    f.wq = Wq;
    f.wsf = Wsf;
    f.flips = flips;
    f.N = static_cast<int32_t>(N);
    f.K = static_cast<int32_t>(K);
    f.sweeps = sweeps;
    f.had_block = b;
    // rows per CTA x columns per thread: 64 float64 sums per thread, shared memory within 227 KB
    if (K <= 2048) return launch_flip<8, 8>(f, dev.sms, st);
    if (K <= 4096) return launch_flip<16, 4>(f, dev.sms, st);
    if (K <= 8192) return launch_flip<32, 2>(f, dev.sms, st);
    return launch_flip<64, 1>(f, dev.sms, st);
}

// ------------------------------------------------------------------------ MoE combine
macaq_status moe_combine(const void *Y, int64_t y_rows, int64_t N, const int32_t *pos, const float *w, int64_t T,
                         int32_t topk, void *out, int32_t out_dtype, cudaStream_t st) {
    if (y_rows < 0 || N <= 0 || N % 8 != 0 || T < 0 || topk < 1 || topk > 1024) return MACAQ_ERR_SHAPE;
    if (N >= (int64_t(1) << 31) || T * topk >= (int64_t(1) << 40)) return MACAQ_ERR_SHAPE;
    if (out_dtype != MACAQ_OUT_BF16 && out_dtype != MACAQ_OUT_F32) return MACAQ_ERR_INVALID_ARG;
    if (T == 0) return MACAQ_OK;
    if ((Y == nullptr && y_rows > 0) || pos == nullptr || w == nullptr || out == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(Y) || !aligned16(out) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
        (reinterpret_cast<uintptr_t>(w) & 3u))
        return MACAQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    macaq_status s = device_info(&dev);
    if (s != MACAQ_OK) return s;
    CombineArgs c;
    c.y = static_cast<const uint16_t *>(Y);
    c.pos = pos;
    c.w = w;
    c.out = out;
    c.y_rows = y_rows;
    c.T = T;
    c.topk = topk;
    c.N = static_cast<int32_t>(N);
    c.out_f32 = out_dtype == MACAQ_OUT_F32;
    const int64_t threads = T * (N / 8);
    int64_t blocks = (threads + kCombineThreads - 1) / kCombineThreads;
    const int64_t cap = static_cast<int64_t>(dev.sms) * 8;   // 8 resident CTAs per SM, grid-stride beyond
    if (blocks > cap) blocks = cap;
    return launch(moe_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kCombineThreads), 0, st, 1, c);
}

}  // namespace macaq

// ============================================================================ C ABI
extern "C" {

const char *macaq_status_str(int status) {
    switch (status) {
        case MACAQ_OK: return "MACAQ_OK";
        case MACAQ_ERR_INVALID_ARG: return "MACAQ_ERR_INVALID_ARG";
        case MACAQ_ERR_SHAPE: return "MACAQ_ERR_SHAPE";
        case MACAQ_ERR_ALIGNMENT: return "MACAQ_ERR_ALIGNMENT";
        case MACAQ_ERR_UNSUPPORTED: return "MACAQ_ERR_UNSUPPORTED";
        case MACAQ_ERR_CUDA: return "MACAQ_ERR_CUDA";
        case MACAQ_ERR_TIMEOUT: return "MACAQ_ERR_TIMEOUT";
        case MACAQ_ERR_WORKSPACE: return "MACAQ_ERR_WORKSPACE";
        default: return "MACAQ_ERR_UNKNOWN";
    }
}

int macaq_last_cuda_error(void) { return macaq::t_last_cuda_error; }

size_t macaq_sf_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0 || K % 128 != 0) return 0;
    return static_cast<size_t>((rows + 127) / 128) * 128 * static_cast<size_t>(K / 32);
}

size_t macaq_grouped_sf_bytes(int64_t total_rows, int32_t E, int64_t K) {
    if (total_rows < 0 || E < 0 || K <= 0 || K % 128 != 0) return 0;
    return static_cast<size_t>((total_rows + 127) / 128 + E) * 128 * static_cast<size_t>(K / 32);
}

size_t macaq_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t E) {
    if (E != 0 || M <= 0 || M > macaq::kSkinnyMaxM || N <= 0 || N % 128 != 0 || K <= 0 || K % 256 != 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    const macaq::SkinnyPlan p = macaq::skinny_plan_cached(M, N, K, sms);
    return p.ok ? p.partial_bytes + p.count_bytes : 0;
}

size_t macaq_fused_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t E) {
    if (M < 0 || N <= 0 || N % 128 != 0 || K <= 0 || K % 128 != 0 || E < 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return macaq::fused_layout(M, N, K, E, sms).total;
}

macaq_status macaq_prep_weights(const void *W, const float *s, int64_t N, int64_t K, int32_t had_block, uint8_t *Wq,
                                uint8_t *Wsf, float *inv_s, macaq_stream_t stream) {
    if (N % 128 != 0) return MACAQ_ERR_SHAPE;
    return macaq::quantize(W, s, N, K, had_block, true, nullptr, 0, Wq, Wsf, s ? inv_s : nullptr,
                           static_cast<cudaStream_t>(stream));
}

macaq_status macaq_act_quant(const void *X, const float *inv_s, int64_t M, int64_t K, int32_t had_block,
                             const int32_t *group_offsets, int32_t E, uint8_t *Xq, uint8_t *Xsf,
                             macaq_stream_t stream) {
    return macaq::quantize(X, inv_s, M, K, had_block, false, group_offsets, E, Xq, Xsf, nullptr,
                           static_cast<cudaStream_t>(stream));
}

macaq_status macaq_act_quant_gather(const void *X, int64_t x_rows, const int32_t *row_index, const float *inv_s,
                                    int64_t M, int64_t K, int32_t had_block, const int32_t *group_offsets, int32_t E,
                                    uint8_t *Xq, uint8_t *Xsf, macaq_stream_t stream) {
    if (row_index == nullptr && M > 0) return MACAQ_ERR_INVALID_ARG;
    if (M == 0) return macaq::quantize(X, inv_s, 0, K, had_block, false, group_offsets, E, Xq, Xsf, nullptr,
                                       static_cast<cudaStream_t>(stream));
    return macaq::quantize(X, inv_s, M, K, had_block, false, group_offsets, E, Xq, Xsf, nullptr,
                           static_cast<cudaStream_t>(stream), row_index, x_rows);
}

macaq_status macaq_act_transform(const void *X, const float *inv_s, int64_t M, int64_t K, int32_t had_block, void *Xt,
                                 macaq_stream_t stream) {
    return macaq::act_transform(X, inv_s, M, K, had_block, Xt, static_cast<cudaStream_t>(stream));
}

size_t macaq_linear_w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    const macaq::WonlyLayout l = macaq::wonly_layout(M, N, K, sms);
    return l.ok ? l.total : 0;
}

macaq_status macaq_linear_w4a16(const void *X, const float *inv_s, int64_t M, int64_t N, int64_t K, int32_t had_block,
                                const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype, void *workspace,
                                size_t ws_bytes, macaq_stream_t stream) {
    return macaq::linear_w4a16(X, inv_s, M, N, K, had_block, Wq, Wsf, Y, out_dtype, workspace, ws_bytes,
                               static_cast<cudaStream_t>(stream));
}

size_t macaq_linear_swiglu_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N <= 0 || N % 256 != 0 || K <= 0 || K % 128 != 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return macaq::swiglu_layout(M, N, K, sms).total;
}

macaq_status macaq_linear_swiglu(const uint8_t *A, const uint8_t *Asf, int64_t M, int64_t N, int64_t K,
                                 const uint8_t *Wq, const uint8_t *Wsf, const float *inv_s_down, int32_t had_block_down,
                                 uint8_t *Hq, uint8_t *Hsf, void *workspace, size_t ws_bytes, macaq_stream_t stream) {
    return macaq::linear_swiglu(A, Asf, M, N, K, Wq, Wsf, inv_s_down, had_block_down, Hq, Hsf, workspace, ws_bytes,
                                static_cast<cudaStream_t>(stream));
}

macaq_status macaq_swiglu_act_quant(const float *GU, int64_t M, int64_t I, const float *inv_s, int32_t had_block,
                                    uint8_t *Hq, uint8_t *Hsf, macaq_stream_t stream) {
    return macaq::swiglu_quant(GU, M, I, inv_s, had_block, Hq, Hsf, static_cast<cudaStream_t>(stream));
}

macaq_status macaq_flip_refine(const void *W, const float *s, int64_t N, int64_t K, int32_t had_block, const float *H,
                               int32_t sweeps, uint8_t *Wq, const uint8_t *Wsf, int32_t *flips, macaq_stream_t stream) {
    return macaq::flip_refine(W, s, N, K, had_block, H, sweeps, Wq, Wsf, flips, static_cast<cudaStream_t>(stream));
}

macaq_status macaq_moe_combine(const void *Y, int64_t y_rows, int64_t N, const int32_t *pos, const float *weights,
                               int64_t T, int32_t topk, void *out, int32_t out_dtype, macaq_stream_t stream) {
    return macaq::moe_combine(Y, y_rows, N, pos, weights, T, topk, out, out_dtype, static_cast<cudaStream_t>(stream));
}

macaq_status macaq_linear(int32_t mode, const void *A, const uint8_t *Asf, const float *inv_s, int64_t M, int64_t N,
                          int64_t K, int32_t had_block, const uint8_t *Wq, const uint8_t *Wsf, void *Y,
                          int32_t out_dtype, void *workspace, size_t ws_bytes, macaq_stream_t stream) {
    if (mode == MACAQ_A_BF16_FUSED || mode == MACAQ_A_BF16_ONE_LAUNCH)
        return macaq::linear_fused(A, inv_s, had_block, nullptr, 0, M, N, K, Wq, Wsf, Y, out_dtype, workspace, ws_bytes,
                                   static_cast<cudaStream_t>(stream), mode == MACAQ_A_BF16_ONE_LAUNCH);
    if (mode != MACAQ_A_QUANTIZED) return MACAQ_ERR_INVALID_ARG;
    return macaq::gemm(static_cast<const uint8_t *>(A), Asf, nullptr, 1, M, N, K, Wq, Wsf, Y, out_dtype, workspace,
                       ws_bytes, static_cast<cudaStream_t>(stream));
}

macaq_status macaq_linear_fixed_scratch(int32_t mode, const void *A, const uint8_t *Asf, const float *inv_s,
                                        int64_t M, int64_t N, int64_t K, int32_t had_block, const uint8_t *Wq,
                                        const uint8_t *Wsf, void *Y, int32_t out_dtype, macaq_stream_t stream) {
    (void)inv_s, (void)had_block;
    if (mode == MACAQ_A_BF16_FUSED || mode == MACAQ_A_BF16_ONE_LAUNCH) return MACAQ_ERR_UNSUPPORTED;
    if (mode != MACAQ_A_QUANTIZED) return MACAQ_ERR_INVALID_ARG;
    return macaq::linear_fixed_scratch(static_cast<const uint8_t *>(A), Asf, M, N, K, Wq, Wsf, Y, out_dtype,
                                       static_cast<cudaStream_t>(stream));
}

macaq_status macaq_grouped_linear(int32_t mode, const void *A, const uint8_t *Asf, const float *inv_s,
                                  const int32_t *group_offsets, int32_t E, int64_t total_rows, int64_t N, int64_t K,
                                  int32_t had_block, const uint8_t *Wq, const uint8_t *Wsf, void *Y,
                                  int32_t out_dtype, void *workspace, size_t ws_bytes, macaq_stream_t stream) {
    if (group_offsets == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (mode == MACAQ_A_BF16_FUSED || mode == MACAQ_A_BF16_ONE_LAUNCH)
        return macaq::linear_fused(A, inv_s, had_block, group_offsets, E, total_rows, N, K, Wq, Wsf, Y, out_dtype,
                                   workspace, ws_bytes, static_cast<cudaStream_t>(stream));
    if (mode != MACAQ_A_QUANTIZED) return MACAQ_ERR_INVALID_ARG;
    return macaq::gemm(static_cast<const uint8_t *>(A), Asf, group_offsets, E, total_rows, N, K, Wq, Wsf, Y,
                       out_dtype, nullptr, 0, static_cast<cudaStream_t>(stream));
}

macaq_status macaq_check_group_offsets(const int32_t *host_offsets, int32_t E, int64_t total_rows) {
    if (host_offsets == nullptr) return MACAQ_ERR_INVALID_ARG;
    if (E < 1 || E > 16384 || total_rows < 0) return MACAQ_ERR_SHAPE;
    if (host_offsets[0] != 0 || static_cast<int64_t>(host_offsets[E]) != total_rows) return MACAQ_ERR_SHAPE;
    for (int32_t e = 0; e < E; ++e)
        if (host_offsets[e + 1] < host_offsets[e]) return MACAQ_ERR_SHAPE;
    return MACAQ_OK;
}

macaq_status macaq_device_status(int32_t *status_out, int32_t reset) {
    if (status_out == nullptr) return MACAQ_ERR_INVALID_ARG;
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, macaq::g_device_status, sizeof v);
    if (e != cudaSuccess) return macaq::cuda_fail(e);
    *status_out = v;
    if (reset) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(macaq::g_device_status, &zero, sizeof zero);
        if (e != cudaSuccess) return macaq::cuda_fail(e);
    }
    return MACAQ_OK;
}

void macaq_set_wait_limit_ns(uint64_t ns) { macaq::g_wait_limit_ns.store(ns ? ns : macaq::kDefaultWaitNs); }

}  // extern "C"
