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
// Data movement: the bf16 input is viewed as a flat array of 128-byte lines and streamed through
// shared memory by TMA (16 KB tiles = 256 groups, 128-byte swizzle so that each thread's 64-byte
// group is read without bank conflicts), in a 4-stage mbarrier ring per CTA; one thread owns one
// group, so the Hadamard stages up to b = 32 stay in registers and b = 64 / 128 add one / two
// shuffle stages with the neighbouring lanes. Codes go out as one 16-byte store per group; four
// neighbouring lanes combine their E8M0 bytes into one 32-bit store in the tiled SF layout.
#pragma once

#include "groups.cuh"
#include "ptx.cuh"

namespace macaq {

constexpr int kQThreads = 256;
constexpr int kQGroupsPerTile = 256;                 // one group per thread
constexpr int kQTileBytes = kQGroupsPerTile * 64;    // 16 KB of bf16
constexpr int kQTileLines = kQTileBytes / 128;       // 128-byte lines per tile (TMA box height)
constexpr int kQStages = 4;

struct QuantArgs {
    const float *mul;         // [K] or [E, K] per-channel multiplier, or nullptr
    const int32_t *offsets;   // [E + 1] grouped row offsets, or nullptr (dense)
    uint8_t *q;               // [rows, K/2] codes
    uint8_t *sf;              // tiled scale factors
    float *inv_s;             // weights: receives 1/mul (IEEE division), or nullptr
    int64_t rows;
    uint32_t K;
    uint32_t kg;              // K / 32
    uint32_t total_groups;    // rows * K / 32
    uint32_t num_tiles;
    int32_t E;                // groups (experts); 1 for a dense call
    uint64_t wait_limit_ns;
};

__host__ __device__ constexpr size_t quant_smem_bytes(int E) {
    return 1024 + static_cast<size_t>(kQStages) * kQTileBytes + 2 * sizeof(int32_t) * (E + 1);
}

template <int kB>
__device__ __forceinline__ void fwht_in_thread(float (&x)[32]) {
    constexpr int kLim = kB < 32 ? kB : 32;
#pragma unroll
    for (int h = 1; h < kLim; h <<= 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if ((j & h) == 0) {
                const float u = x[j], w = x[j + h];
                x[j] = __fadd_rn(u, w);
                x[j + h] = __fsub_rn(u, w);
            }
        }
    }
}

// One cross-lane butterfly stage: this lane's group is paired with lane ^ lane_bit's group.
__device__ __forceinline__ void fwht_cross_lane(float (&x)[32], int lane_bit) {
    const bool upper = (threadIdx.x & lane_bit) != 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float o = __shfl_xor_sync(0xffffffffu, x[j], lane_bit);
        x[j] = upper ? __fsub_rn(o, x[j]) : __fadd_rn(x[j], o);
    }
}

template <int kB, bool kWeight>
__global__ void __launch_bounds__(kQThreads) quant_kernel(const __grid_constant__ CUtensorMap xmap, QuantArgs a) {
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[kQStages];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    int32_t *s_off = reinterpret_cast<int32_t *>(tiles + kQStages * kQTileBytes);
    int32_t *s_tb = s_off + (a.E + 1);

    const int tid = threadIdx.x;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kQStages; ++s) mbar_init(&full_bar[s], 1);
        fence_mbar_init();
        if (a.num_tiles > 0) prefetch_tensor_map(&xmap);
    }
    load_group_layout(a.offsets, a.E, a.rows, s_off, s_tb);  // contains __syncthreads

    // prologue: the first kQStages-1 tiles of this CTA
    if (tid == 0) {
        for (int s = 0; s < kQStages - 1; ++s) {
            const uint32_t t = blockIdx.x + s * gridDim.x;
            if (t < a.num_tiles) {
                mbar_arrive_expect_tx(&full_bar[s], kQTileBytes);
                tma_load_2d(tiles + s * kQTileBytes, &xmap, &full_bar[s], 0, static_cast<int32_t>(t * kQTileLines));
            }
        }
    }

    uint32_t it = 0;
    bool ok = true;
    for (uint32_t t = blockIdx.x; t < a.num_tiles; t += gridDim.x, ++it) {
        const int s = it % kQStages;
        const bool ready = mbar_wait(&full_bar[s], (it / kQStages) & 1, a.wait_limit_ns);
        // every thread is done with tile it-1 and tile it has landed
        if (!__syncthreads_and(ready)) {
            ok = false;
            break;
        }
        if (tid == 0) {
            const uint32_t tn = t + (kQStages - 1) * gridDim.x;
            if (tn < a.num_tiles) {
                const int sn = (it + kQStages - 1) % kQStages;  // the stage tile it-1 used
                mbar_arrive_expect_tx(&full_bar[sn], kQTileBytes);
                tma_load_2d(tiles + sn * kQTileBytes, &xmap, &full_bar[sn], 0, static_cast<int32_t>(tn * kQTileLines));
            }
        }

        const uint32_t gi = t * kQGroupsPerTile + tid;  // global group index
        const bool valid = gi < a.total_groups;
        const uint32_t m = valid ? gi / a.kg : 0;
        const uint32_t g = valid ? gi - m * a.kg : 0;
        const int e = valid ? find_group(s_off, a.E, m) : -1;

        // 64 bytes of this group from the swizzled tile: line tid/2, logical chunks (tid&1)*4 + i
        const uint8_t *line = tiles + s * kQTileBytes + (tid >> 1) * 128;
        float x[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int phys = (((tid & 1) << 2) + i) ^ ((tid >> 1) & 7);
            const uint4 v = *reinterpret_cast<const uint4 *>(line + phys * 16);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                x[8 * i + 2 * p] = __uint_as_float(w[p] << 16);
                x[8 * i + 2 * p + 1] = __uint_as_float(w[p] & 0xFFFF0000u);
            }
        }

        if (a.mul != nullptr) {
            const int eg = e < 0 ? 0 : e;
            const float4 *mp = reinterpret_cast<const float4 *>(a.mul + static_cast<uint64_t>(eg) * a.K + g * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 mv = __ldg(mp + i);
                x[4 * i + 0] = __fmul_rn(x[4 * i + 0], mv.x);
                x[4 * i + 1] = __fmul_rn(x[4 * i + 1], mv.y);
                x[4 * i + 2] = __fmul_rn(x[4 * i + 2], mv.z);
                x[4 * i + 3] = __fmul_rn(x[4 * i + 3], mv.w);
            }
        }

        if constexpr (kB > 1) {
            fwht_in_thread<kB>(x);
            if constexpr (kB >= 64) fwht_cross_lane(x, 1);
            if constexpr (kB >= 128) fwht_cross_lane(x, 2);
            if constexpr (kWeight) {
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = __fmul_rn(x[j], 1.0f / kB);
            }
        }

        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(x[j]));
        const int ef = static_cast<int>(__float_as_uint(amax) >> 23);  // biased exponent (amax >= 0)
        const uint32_t E8 = static_cast<uint32_t>(ef > 2 ? ef - 2 : 0);
        const float inv_scale = __uint_as_float((254u - E8) << 23);   // 2^(127 - E), a normal float

#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = __fmul_rn(x[j], inv_scale);
        uint4 packed;
        packed.x = cvt_e2m1x8(x + 0);
        packed.y = cvt_e2m1x8(x + 8);
        packed.z = cvt_e2m1x8(x + 16);
        packed.w = cvt_e2m1x8(x + 24);
        const bool store = valid && e >= 0;
        if (store) *reinterpret_cast<uint4 *>(a.q + static_cast<uint64_t>(gi) * 16) = packed;

        // lanes 4i..4i+3 hold scale columns 4c..4c+3 of one row: one 32-bit store
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, E8, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, E8, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, E8, 3);
        if (store && (lane & 3) == 0) {
            const uint32_t sf_row = static_cast<uint32_t>(s_tb[e]) * 128 + (m - static_cast<uint32_t>(s_off[e]));
            *reinterpret_cast<uint32_t *>(a.sf + sf_offset(sf_row, g, a.kg >> 2)) =
                E8 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
    }

    if (!ok) {
        // a tile never arrived: wait (bounded) for the copies this CTA still has in flight
        if (tid == 0) {
            for (uint32_t j = it; j < it + kQStages - 1; ++j) {
                const uint32_t tj = blockIdx.x + j * gridDim.x;
                if (tj >= a.num_tiles) break;
                if (!mbar_wait(&full_bar[j % kQStages], (j / kQStages) & 1, 2000000000ull)) break;
            }
        }
        return;
    }

    // zero the scale factors of every group's padding rows (rows M_e .. 128 * tiles_e - 1)
    const uint32_t kq = a.kg >> 2;
    for (int e = blockIdx.x; e < a.E; e += gridDim.x) {
        const uint32_t me = static_cast<uint32_t>(s_off[e + 1] - s_off[e]);
        const uint32_t nt = static_cast<uint32_t>(s_tb[e + 1] - s_tb[e]);
        const uint32_t words = (nt * 128 - me) * kq;
        for (uint32_t w = tid; w < words; w += blockDim.x) {
            const uint32_t pr = me + w / kq;
            const uint32_t c4 = (w - (w / kq) * kq) * 4;
            const uint32_t sf_row = static_cast<uint32_t>(s_tb[e]) * 128 + pr;
            *reinterpret_cast<uint32_t *>(a.sf + sf_offset(sf_row, c4, kq)) = 0u;
        }
    }

    if (kWeight && a.inv_s != nullptr && a.mul != nullptr) {
        for (uint32_t k = blockIdx.x * blockDim.x + tid; k < a.K; k += gridDim.x * blockDim.x)
            a.inv_s[k] = __fdiv_rn(1.0f, a.mul[k]);
    }
}

}  // namespace macaq
