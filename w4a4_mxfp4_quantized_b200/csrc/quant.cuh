// quant.cuh -- the transform + MXFP4 quantization kernel (activations online, weights offline).
//
// Per 32-element group of a row, in fp32 and in this exact order (bit-identical to the
// plain definition):
//   v[k] = fl32(x[k] * mul[k])               mul = 1/s (activations) or s (weights); absent = 1
//   v    = v * H_b on each aligned block     butterfly stages h = 1, 2, ..., b/2 (Sylvester H_b)
//   v[k] = v[k] * (1/b)                      weights only (exact: a power of two)
//   E    = clamp(floor(log2 max|v|) - 2 + 127, 0, 254)            OCP MX v1.0 shared exponent
//   code = E2M1_rne_satfinite(v[k] * 2^(127-E)), two codes per byte, even k in the low nibble
// Sources: aipolix.com page on MACaQ (Persian), paragraphs 2-3; OCP Microscaling Formats v1.0.
//
// Data movement: the bf16 input is cut into tiles of (256 / w) rows x w groups (w = 32, 16, 8 or 4
// groups, the largest that divides K/32), always 16 KB, streamed through shared memory by TMA with
// the 128-byte swizzle (each thread's 64-byte group is read without bank conflicts). One thread owns
// one group; the Hadamard stages up to b = 32 stay in registers (packed fp32 pairs), b = 64 / 128 add
// one / two shuffle stages with the neighbouring lanes. Codes go out as one 16-byte store per group;
// four neighbouring lanes combine their E8M0 bytes into one 32-bit store in the tiled SF layout.
#pragma once

#include <cuda_bf16.h>

#include "groups.cuh"
#include "ptx.cuh"

namespace macaq {

constexpr int kQConsumerWarps = 8;
constexpr int kQConsumers = kQConsumerWarps * 32;    // one 32-element group per consumer thread per tile
constexpr int kQThreads = kQConsumers + 32;          // + one producer warp
constexpr int kQTileBytes = kQConsumers * 64;        // 16 KB of bf16
constexpr int kQStages = 4;

struct QuantArgs {
    const float *mul;         // [K] or [E, K] per-channel multiplier, or nullptr
    const int32_t *offsets;   // [E + 1] grouped row offsets, or nullptr (dense)
    uint8_t *q;               // [rows, K/2] codes
    uint8_t *sf;              // tiled scale factors
    float *inv_s;             // weights: receives 1/mul (IEEE division), or nullptr
    int64_t rows;
    uint32_t K;
    uint32_t kg;              // K / 32 groups per row
    uint32_t slab_groups;     // groups per column slab: 32, 16, 8 or 4 (divides kg)
    uint32_t slab_shift;      // log2(slab_groups)
    uint32_t slabs;           // kg / slab_groups
    uint32_t tile_rows;       // rows per tile = 256 / slab_groups
    uint32_t row_tiles;       // ceil(rows / tile_rows)
    int32_t E;                // groups (experts); 1 for a dense call
    uint64_t wait_limit_ns;
};

__host__ __device__ constexpr size_t quant_smem_bytes(int E) {
    return 1024 + static_cast<size_t>(kQStages) * kQTileBytes + 2 * sizeof(int32_t) * (E + 1);
}

// The 32 values of a group live in 16 packed pairs p[i] = (v[2i], v[2i+1]).
// Butterfly stage h = 1 pairs the two lanes of one register; stages h >= 2 pair register i with
// register i + h/2 lane by lane, so they run as packed adds/subtracts.
template <int kB>
__device__ __forceinline__ void fwht_in_thread(uint64_t (&p)[16]) {
    if constexpr (kB >= 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float a, c;
            upk2(p[i], a, c);
            p[i] = pk2(__fadd_rn(a, c), __fsub_rn(a, c));
        }
    }
    constexpr int kLim = (kB < 32 ? kB : 32) / 2;  // stages h = 2 .. min(b, 32)/2, as h/2
#pragma unroll
    for (int hp = 1; hp < kLim; hp <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & hp) == 0) {
                const uint64_t a = p[i], c = p[i + hp];
                p[i] = add2(a, c);
                p[i + hp] = sub2(a, c);
            }
        }
    }
}

// One cross-lane butterfly stage: this lane's group is paired with lane ^ lane_bit's group
// (the next group of the same row).
__device__ __forceinline__ void fwht_cross_lane(uint64_t (&p)[16], int lane_bit) {
    const bool upper = (threadIdx.x & lane_bit) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, p[i], lane_bit);
        p[i] = upper ? sub2(o, p[i]) : add2(p[i], o);
    }
}

__device__ __forceinline__ void load_mul(const float *mul, uint64_t (&mv)[16]) {
    const float4 *mp = reinterpret_cast<const float4 *>(mul);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 f = __ldg(mp + i);
        mv[2 * i] = pk2(f.x, f.y);
        mv[2 * i + 1] = pk2(f.z, f.w);
    }
}

// Hadamard stages (and, for weights, the exact 1/b) on one 32-element group held as 16 packed fp32
// pairs, then its MXFP4 encoding: the 16 code bytes (even k in the low nibble) and the E8M0
// exponent. For b >= 64 the group is paired with the groups of lanes lane ^ 1 (and lane ^ 2), which
// hold the next groups of the same row: the whole warp calls it together.
// OCP MX v1.0 encoding of one 32-element group held as 16 packed fp32 pairs: the shared E8M0
// exponent E = clamp(floor(log2 amax) - 2 + 127, 0, 254) read from the exponent field of amax, and
// the 32 E2M1 codes of v * 2^(127 - E) (round to nearest even, saturating), two per byte.
__device__ __forceinline__ void mx_encode_group(const uint64_t (&p)[16], uint4 &packed, uint32_t &E8);

template <int kB, bool kWeight>
__device__ __forceinline__ void transform_quantize_group(uint64_t (&p)[16], uint4 &packed, uint32_t &E8) {
    if constexpr (kB > 1) {
        fwht_in_thread<kB>(p);
        if constexpr (kB >= 64) fwht_cross_lane(p, 1);
        if constexpr (kB >= 128) fwht_cross_lane(p, 2);
        if constexpr (kWeight) {
            const uint64_t inv_b = pk2(1.0f / kB, 1.0f / kB);
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], inv_b);
        }
    }
    mx_encode_group(p, packed, E8);
}

__device__ __forceinline__ void mx_encode_group(const uint64_t (&p)[16], uint4 &packed, uint32_t &E8) {
    float mx[16];  // max |v| as a tree: short dependency chains
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float lo, hi;
        upk2(p[i], lo, hi);
        mx[i] = fmaxf(fabsf(lo), fabsf(hi));
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
    const int ef = static_cast<int>(__float_as_uint(mx[0]) >> 23);  // biased exponent (amax >= 0)
    E8 = static_cast<uint32_t>(ef > 2 ? ef - 2 : 0);
    const float inv_scale = __uint_as_float((254u - E8) << 23);     // 2^(127 - E), a normal float
    const uint64_t inv_scale2 = pk2(inv_scale, inv_scale);

    float y[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) upk2(mul2(p[i], inv_scale2), y[2 * i], y[2 * i + 1]);
    packed.x = cvt_e2m1x8(y + 0);
    packed.y = cvt_e2m1x8(y + 8);
    packed.z = cvt_e2m1x8(y + 16);
    packed.w = cvt_e2m1x8(y + 24);
}

// Unpacks 32 bf16 (four 16-byte words, element order) into 16 packed fp32 pairs.
__device__ __forceinline__ void unpack_bf16x32(const uint4 (&raw)[4], uint64_t (&p)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        p[4 * i + 0] = pk2(__uint_as_float(raw[i].x << 16), __uint_as_float(raw[i].x & 0xFFFF0000u));
        p[4 * i + 1] = pk2(__uint_as_float(raw[i].y << 16), __uint_as_float(raw[i].y & 0xFFFF0000u));
        p[4 * i + 2] = pk2(__uint_as_float(raw[i].z << 16), __uint_as_float(raw[i].z & 0xFFFF0000u));
        p[4 * i + 3] = pk2(__uint_as_float(raw[i].w << 16), __uint_as_float(raw[i].w & 0xFFFF0000u));
    }
}

// The rest of one group's work once its 32 inputs are fp32 pairs in registers: the per-channel
// multiply (mv, when a.mul is set), Hadamard and MXFP4 (transform_quantize_group), the 16 code bytes
// of row m, and the E8M0 byte, which lanes 4i..4i+3 (scale columns 4c..4c+3 of one row) combine into
// one 32-bit store in the tiled layout. e < 0 marks a row outside every group: nothing is stored.
// The whole warp calls it together (shuffles).
template <int kB, bool kWeight>
__device__ __forceinline__ void quantize_store_group(uint64_t (&p)[16], const uint64_t (&mv)[16], bool with_mul,
                                                     const QuantArgs &a, int e, uint32_t m, uint32_t g,
                                                     const int32_t *s_off, const int32_t *s_tb, int lane) {
    if (with_mul) {
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], mv[i]);
    }
    uint4 packed;
    uint32_t E8;
    transform_quantize_group<kB, kWeight>(p, packed, E8);
    const bool store = e >= 0;
    if (store) *reinterpret_cast<uint4 *>(a.q + static_cast<uint64_t>(m) * (a.K / 2) + g * 16) = packed;
    const uint32_t b1 = __shfl_down_sync(0xffffffffu, E8, 1);
    const uint32_t b2 = __shfl_down_sync(0xffffffffu, E8, 2);
    const uint32_t b3 = __shfl_down_sync(0xffffffffu, E8, 3);
    if (store && (lane & 3) == 0) {
        const uint32_t sf_row = static_cast<uint32_t>(s_tb[e]) * 128 + (m - static_cast<uint32_t>(s_off[e]));
        *reinterpret_cast<uint32_t *>(a.sf + sf_offset(sf_row, g, a.kg >> 2)) = E8 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
}

// The weight-only path's activation transform of one group: the per-channel multiply, the Hadamard
// stages (activations: no 1/b), then each value rounded to bf16 (nearest even); the 64 bytes go to
// row m, group g of a bf16 [rows, K] output (a.q reinterpreted). The whole warp calls it (shuffles).
template <int kB>
__device__ __forceinline__ void transform_store_bf16_group(uint64_t (&p)[16], const uint64_t (&mv)[16], bool with_mul,
                                                           const QuantArgs &a, bool store, uint32_t m, uint32_t g) {
    if (with_mul) {
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], mv[i]);
    }
    if constexpr (kB > 1) {
        fwht_in_thread<kB>(p);
        if constexpr (kB >= 64) fwht_cross_lane(p, 1);
        if constexpr (kB >= 128) fwht_cross_lane(p, 2);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(a.q + (static_cast<uint64_t>(m) * a.K + g * 32) * 2);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float lo, hi;
            upk2(p[4 * i + k], lo, hi);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
            w[k] = *reinterpret_cast<uint32_t *>(&b2);
        }
        if (store) dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Zeroes the scale factors of every group's padding rows (rows M_e .. 128 * tiles_e - 1, all in the
// group's last 128-row tile). Work items are (group, 128x4 scale tile of that last row tile), dealt to
// the warps of all CTAs; a warp writes the tile's 128 words with four coalesced 128-byte stores, each
// lane zeroing its word only when the word's row is a padding row (word w holds row
// (w % 4) * 32 + w / 4), so the words of valid rows are never touched.
__device__ __forceinline__ void zero_sf_padding(const QuantArgs &a, const int32_t *s_off, const int32_t *s_tb, int warp,
                                                int lane, int warps) {
    const uint32_t kq = a.kg >> 2;
    const uint32_t items = static_cast<uint32_t>(a.E) * kq;
    for (uint32_t it = blockIdx.x * warps + warp; it < items; it += gridDim.x * warps) {
        const uint32_t e = it / kq, ct = it - e * kq;
        const uint32_t me = static_cast<uint32_t>(s_off[e + 1] - s_off[e]);
        const uint32_t nt = static_cast<uint32_t>(s_tb[e + 1] - s_tb[e]);
        if (nt == 0 || me == nt * 128) continue;
        const uint32_t first = (nt - 1) * 128;   // the last tile's first row, counted inside the group
        uint32_t *tile = reinterpret_cast<uint32_t *>(a.sf + sf_offset((static_cast<uint32_t>(s_tb[e]) + nt - 1) * 128, 4 * ct, kq));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w = j * 32 + lane;
            if (first + (w & 3) * 32 + (w >> 2) >= me) tile[w] = 0u;
        }
    }
}

// Work split: the K axis is cut into column slabs of slab_groups groups; a tile is tile_rows rows of
// one slab (always 256 groups, 16 KB). A CTA keeps one slab for its whole life and walks a
// contiguous run of its row tiles, so each consumer thread owns one fixed group column and keeps that
// column's 32 multipliers in registers (reloaded only where the expert changes). A producer warp streams the tiles with TMA (3-D tensor map rows x 128-byte chunks x
// 64 elements, 128-byte swizzle) into a 4-stage ring with full/empty mbarriers.
template <int kB, bool kWeight, bool kBf16Out = false>
__global__ void __launch_bounds__(kQThreads, 2) quant_kernel(const __grid_constant__ CUtensorMap xmap, QuantArgs a) {
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[kQStages];
    __shared__ uint64_t empty_bar[kQStages];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    int32_t *s_off = reinterpret_cast<int32_t *>(tiles + kQStages * kQTileBytes);
    int32_t *s_tb = s_off + (a.E + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t slab = blockIdx.x % a.slabs;
    const uint32_t ctas_per_slab = gridDim.x / a.slabs;
    // each CTA takes a contiguous run of its slab's row tiles, so the expert (and with it the
    // per-channel multipliers a thread keeps in registers) changes only at expert boundaries
    const uint32_t c_in_slab = blockIdx.x / a.slabs;
    const uint32_t rt_begin = static_cast<uint32_t>(static_cast<uint64_t>(a.row_tiles) * c_in_slab / ctas_per_slab);
    const uint32_t rt_end = static_cast<uint32_t>(static_cast<uint64_t>(a.row_tiles) * (c_in_slab + 1) / ctas_per_slab);

    if (tid == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kQConsumerWarps);
        }
        fence_mbar_init();
        if (rt_begin < rt_end) prefetch_tensor_map(&xmap);
    }
    griddep_wait();  // X, the multipliers, the offsets and the outputs may belong to the previous kernel
    load_group_layout(a.offsets, a.E, a.rows, s_off, s_tb);  // contains __syncthreads
    griddep_launch_dependents();

    if (warp == kQConsumerWarps) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            uint32_t j = 0;
            for (uint32_t rt = rt_begin; rt < rt_end; ++rt, ++j) {
                const int s = j % kQStages;
                if (j >= kQStages && !mbar_wait(&empty_bar[s], ((j / kQStages) & 1) ^ 1, a.wait_limit_ns)) break;
                mbar_arrive_expect_tx(&full_bar[s], kQTileBytes);
                tma_load_3d(tiles + s * kQTileBytes, &xmap, &full_bar[s], 0,
                            static_cast<int32_t>(slab * (a.slab_groups / 2)), static_cast<int32_t>(rt * a.tile_rows));
            }
            // let the copies this thread issued land before the CTA can exit
            for (uint32_t i = (j > kQStages ? j - kQStages : 0); i < j; ++i)
                if (!mbar_wait(&full_bar[i % kQStages], (i / kQStages) & 1, 2000000000ull)) break;
        }
    } else {
        // ---------------------------------------------------------------- consumers
        const uint32_t gc = tid & (a.slab_groups - 1);      // group within the slab
        const uint32_t r_in = tid >> a.slab_shift;          // row within the tile
        const uint32_t g = slab * a.slab_groups + gc;       // group column of this thread
        const uint32_t line = r_in * (a.slab_groups / 2) + (gc >> 1);  // 128-byte line of the tile
        uint64_t mv[16];
        int cur_e = -1;
        uint32_t j = 0;
        for (uint32_t rt = rt_begin; rt < rt_end; ++rt, ++j) {
            const int s = j % kQStages;
            const uint32_t m = rt * a.tile_rows + r_in;
            const bool valid = m < a.rows;
            const int e = valid ? find_group(s_off, a.E, m) : -1;
            if (a.mul != nullptr && e != cur_e && e >= 0) {   // per-channel multipliers of this column
                load_mul(a.mul + static_cast<uint64_t>(e) * a.K + g * 32, mv);
                cur_e = e;
            }
            // the whole warp leaves together if any lane's wait ran out (shuffles follow)
            if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[s], (j / kQStages) & 1, a.wait_limit_ns))) break;

            const uint8_t *lp = tiles + s * kQTileBytes + line * 128;
            uint4 raw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int phys = (((gc & 1) << 2) + i) ^ (line & 7);
                raw[i] = *reinterpret_cast<const uint4 *>(lp + phys * 16);
            }
            uint64_t p[16];
            unpack_bf16x32(raw, p);
            // Release the stage only after every lane has its words in registers (the unpacking above
            // consumed them), and order those generic-proxy reads before the next TMA write of the
            // stage, which is an async-proxy access.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[s]);
            if constexpr (kBf16Out) transform_store_bf16_group<kB>(p, mv, a.mul != nullptr, a, e >= 0, m, g);
            else quantize_store_group<kB, kWeight>(p, mv, a.mul != nullptr, a, e, m, g, s_off, s_tb, lane);
        }
    }

    if constexpr (!kBf16Out) zero_sf_padding(a, s_off, s_tb, warp, lane, kQThreads / 32);

    if (kWeight && a.inv_s != nullptr && a.mul != nullptr) {
        for (uint32_t k = blockIdx.x * blockDim.x + tid; k < a.K; k += gridDim.x * blockDim.x)
            a.inv_s[k] = __fdiv_rn(1.0f, a.mul[k]);
    }
}

// Activation quantization with a row gather (MoE dispatch): output row m is the transform and MXFP4
// of input row row_index[m] of X (x_rows rows), so the caller never materialises the expert-sorted
// copy of the activations. Same work split as quant_kernel (column slabs, contiguous runs of row
// tiles, multipliers in registers per expert) and the same per-group arithmetic; the gathered rows
// are not contiguous, so each thread loads its 64-byte group straight from global memory (a warp's
// lanes read one or more whole 512- to 2048-byte row segments), one row tile ahead of the one it
// quantizes. Index values outside [0, x_rows) are clamped into it (no access leaves X; the result
// for such a row is that of the clamped row).
// Source: glonce.com page on MACaQ, paragraph 5 (grouped matmul for mixture-of-experts layers).
struct GatherArgs {
    const uint16_t *x;         // bf16 [x_rows, K]
    const int32_t *row_index;  // [rows]
    int64_t x_rows;
};

__device__ __forceinline__ void load_group_global(const uint16_t *src, uint4 (&raw)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(raw[i].x), "=r"(raw[i].y), "=r"(raw[i].z), "=r"(raw[i].w)
                     : "l"(src + 8 * i));
}

template <int kB>
__global__ void __launch_bounds__(kQConsumers, 2) quant_gather_kernel(QuantArgs a, GatherArgs gx) {
    extern __shared__ uint8_t dsmem[];
    int32_t *s_off = reinterpret_cast<int32_t *>(dsmem);
    int32_t *s_tb = s_off + (a.E + 1);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t slab = blockIdx.x % a.slabs;
    const uint32_t ctas_per_slab = gridDim.x / a.slabs;
    const uint32_t c_in_slab = blockIdx.x / a.slabs;
    const uint32_t rt_begin = static_cast<uint32_t>(static_cast<uint64_t>(a.row_tiles) * c_in_slab / ctas_per_slab);
    const uint32_t rt_end = static_cast<uint32_t>(static_cast<uint64_t>(a.row_tiles) * (c_in_slab + 1) / ctas_per_slab);
    griddep_wait();  // X, the indices, the offsets and the outputs may belong to the previous kernel
    load_group_layout(a.offsets, a.E, a.rows, s_off, s_tb);  // contains __syncthreads
    griddep_launch_dependents();

    const uint32_t gc = tid & (a.slab_groups - 1);
    const uint32_t r_in = tid >> a.slab_shift;
    const uint32_t g = slab * a.slab_groups + gc;
    auto fetch = [&](uint32_t rt, uint4 (&raw)[4]) {
        const uint32_t m = rt * a.tile_rows + r_in;
        if (m < a.rows) {
            int64_t src = gx.row_index[m];
            src = src < 0 ? 0 : (src >= gx.x_rows ? gx.x_rows - 1 : src);
            load_group_global(gx.x + static_cast<uint64_t>(src) * a.K + g * 32, raw);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) raw[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint64_t mv[16];
    int cur_e = -1;
    uint4 next[4];
    if (rt_begin < rt_end) fetch(rt_begin, next);
    for (uint32_t rt = rt_begin; rt < rt_end; ++rt) {
        uint4 raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) raw[i] = next[i];
        if (rt + 1 < rt_end) fetch(rt + 1, next);   // the next tile's loads are in flight meanwhile
        const uint32_t m = rt * a.tile_rows + r_in;
        const int e = m < a.rows ? find_group(s_off, a.E, m) : -1;
        if (a.mul != nullptr && e != cur_e && e >= 0) {
            load_mul(a.mul + static_cast<uint64_t>(e) * a.K + g * 32, mv);
            cur_e = e;
        }
        uint64_t p[16];
        unpack_bf16x32(raw, p);
        quantize_store_group<kB, false>(p, mv, a.mul != nullptr, a, e, m, g, s_off, s_tb, lane);
    }
    zero_sf_padding(a, s_off, s_tb, warp, lane, kQConsumers / 32);
}

}  // namespace macaq
