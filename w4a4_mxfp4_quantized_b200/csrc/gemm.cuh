// gemm.cuh -- block-scaled W4A4 GEMM on the sm_100a tensor cores (tcgen05.mma kind::mxf4).
//
//   Y[m, n] = sum_k (qa[m,k] * 2^(ea[m,k/32]-127)) * (qw[n,k] * 2^(ew[n,k/32]-127))
//
// fp32 accumulation in tensor memory, bf16 (round-to-nearest-even) or fp32 output. Dense and grouped
// (MoE) forms; the grouped form maps each 128-row tile to its expert from the device-side offsets.
// Source: glonce.com page on MACaQ, paragraph 5 (W4A4 dense and grouped matmul kernels).
//
// One CTA computes a 128 x BN output tile. Warp roles (192 threads):
//   warp 0      TMA producer: per K-block of 256 elements, the A tile (128 rows x 128 bytes) and the
//               B tile (BN rows x 128 bytes) with 128-byte swizzle via tensor maps, plus the matching
//               scale-factor tiles (already in the tcgen05 128x4 tiling) by plain bulk copies;
//   warp 1      TMEM allocator and MMA issuer: copies the scale factors into TMEM (tcgen05.cp
//               32x128b.warpx4), then issues 4 MMAs of 128 x BN x 64, and frees the stage with
//               tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld of the fp32 accumulator (each warp reads its 32-lane quarter),
//               conversion and row stores.
// Stages form an mbarrier ring; every wait is bounded and a timeout leaves the kernel cleanly.
#pragma once

#include <cuda_bf16.h>

#include "groups.cuh"
#include "ptx.cuh"

namespace macaq {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 FP4 elements per K-block
constexpr int kGemmThreads = 192;
constexpr uint64_t kDrainLimitNs = 2000000000ull;  // waits for the kernel's own copies / MMAs to land

template <int BN>
struct GemmCfg {
    static constexpr int kStages = BN == 256 ? 4 : 6;
    static constexpr int kABytes = kBM * kBKBytes;
    static constexpr int kBBytes = BN * kBKBytes;
    static constexpr int kSfaBytes = 1024;                 // 128 rows x 8 scale columns
    static constexpr int kSfbBytes = (BN / 128) * 1024;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes;
    static constexpr int kTmemSfa = BN;                    // 2 chunks x 4 columns
    static constexpr int kTmemSfb = BN + 8;                // 2 chunks x (BN / 32) columns
    static constexpr int kTmemUsed = BN + 8 + BN / 16;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                     : kTmemUsed <= 256 ? 256 : 512;
};

struct GemmArgs {
    const uint8_t *asf;        // tiled SF of A (dense: ceil(M/128) tiles; grouped: per-expert tiles)
    const uint8_t *bsf;        // tiled SF of W; expert e at bsf + e * bsf_stride
    void *y;                   // [rows, N] bf16 or fp32
    const int32_t *offsets;    // grouped: [E + 1]; dense: nullptr
    int64_t rows;              // M (dense) or total rows (grouped)
    int32_t N;
    int32_t K;
    int32_t E;                 // experts (1 for dense)
    int32_t out_f32;
    uint64_t bsf_stride;       // bytes between experts' SF
    uint64_t wait_limit_ns;
};

template <int BN>
__host__ __device__ constexpr size_t gemm_smem_bytes(int E) {
    return GemmCfg<BN>::kSmemBytes + 2 * sizeof(int32_t) * (E + 1);
}

template <int BN, bool kGrouped>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_mxf4_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap, GemmArgs g) {
    using C = GemmCfg<BN>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[S];
    __shared__ uint64_t empty_bar[S];
    __shared__ uint64_t accum_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int mma_failed;  // set by the MMA thread when it stops early

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + S * C::kABytes;
    uint8_t *sSfa = sB + S * C::kBBytes;
    uint8_t *sSfb = sSfa + S * C::kSfaBytes;
    int32_t *s_off = reinterpret_cast<int32_t *>(sSfb + S * C::kSfbBytes);
    int32_t *s_tb = s_off + (g.E + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_tile = blockIdx.x;
    const int m_tile = blockIdx.y;

    // ---- which rows this CTA owns
    int64_t row0, row_end;
    int expert = 0;
    if constexpr (kGrouped) {
        load_group_layout(g.offsets, g.E, g.rows, s_off, s_tb);  // block-wide
        if (m_tile >= s_tb[g.E]) return;                         // beyond the last expert's tiles
        int lo = 0, hi = g.E;                                    // s_tb[lo] <= m_tile < s_tb[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_tb[mid] <= m_tile) lo = mid;
            else hi = mid;
        }
        expert = lo;
        row0 = s_off[expert] + static_cast<int64_t>(m_tile - s_tb[expert]) * kBM;
        row_end = s_off[expert + 1];
    } else {
        row0 = static_cast<int64_t>(m_tile) * kBM;
        row_end = g.rows;
    }
    if (row_end > row0 + kBM) row_end = row0 + kBM;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accum_bar, 1);
        mma_failed = 0;
        fence_mbar_init();
        prefetch_tensor_map(&amap);
        prefetch_tensor_map(&bmap);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const int K = g.K;
    const int kq = K / 128;                      // scale tiles per SF row tile
    const int num_kb = (K + 255) / 256;
    const uint64_t limit = g.wait_limit_ns;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer
            const uint8_t *asf = g.asf + static_cast<uint64_t>(m_tile) * kq * 512;
            const uint8_t *bsf = g.bsf + static_cast<uint64_t>(expert) * g.bsf_stride +
                                 static_cast<uint64_t>(n_tile) * (BN / 128) * kq * 512;
            const int32_t brow = expert * g.N + n_tile * BN;
            int kb = 0;
            for (; kb < num_kb; ++kb) {
                const int s = kb % S;
                if (kb >= S && !mbar_wait(&empty_bar[s], ((kb / S) & 1) ^ 1, limit)) break;
                const int kch = (K - kb * 256) >= 256 ? 2 : 1;   // 128-element scale chunks in this block
                mbar_arrive_expect_tx(&full_bar[s], C::kABytes + C::kBBytes + kch * 512 * (1 + BN / 128));
                tma_load_2d(sA + s * C::kABytes, &amap, &full_bar[s], kb * kBKBytes, static_cast<int32_t>(row0));
                tma_load_2d(sB + s * C::kBBytes, &bmap, &full_bar[s], kb * kBKBytes, brow);
                bulk_load(sSfa + s * C::kSfaBytes, asf + kb * 1024, kch * 512, &full_bar[s]);
#pragma unroll
                for (int h = 0; h < BN / 128; ++h)
                    bulk_load(sSfb + s * C::kSfbBytes + h * 1024, bsf + static_cast<uint64_t>(h) * kq * 512 + kb * 1024,
                              kch * 512, &full_bar[s]);
            }
            // let the copies this thread issued land before the CTA can exit
            for (int j = (kb > S ? kb - S : 0); j < kb; ++j)
                if (!mbar_wait(&full_bar[j % S], (j / S) & 1, kDrainLimitNs)) break;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t idesc_lo = idesc_mxf4(BN, 0);  // scale bytes 0-1 of each TMEM column
            const uint32_t idesc_hi = idesc_mxf4(BN, 2);  // scale bytes 2-3
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % S;
                if (!mbar_wait(&full_bar[s], (kb / S) & 1, limit)) {
                    mma_failed = 1;
                    __threadfence_block();
                    break;
                }
                tc_fence_after();
                const int kch = (K - kb * 256) >= 256 ? 2 : 1;
                for (int c = 0; c < kch; ++c) {
                    tc_cp_sf(tmem + C::kTmemSfa + 4 * c, sdesc_sf(smem_u32(sSfa + s * C::kSfaBytes + c * 512)));
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h)
                        tc_cp_sf(tmem + C::kTmemSfb + c * (BN / 32) + 4 * h,
                                 sdesc_sf(smem_u32(sSfb + s * C::kSfbBytes + h * 1024 + c * 512)));
                }
                const uint64_t adesc = sdesc_sw128(smem_u32(sA + s * C::kABytes));
                const uint64_t bdesc = sdesc_sw128(smem_u32(sB + s * C::kBBytes));
                for (int j = 0; j < 2 * kch; ++j) {
                    const int c = j >> 1;
                    // K step j covers bytes [32j, 32j + 32) of every 128-byte row
                    tc_mma_mxf4(tmem, adesc + 2 * j, bdesc + 2 * j, (j & 1) ? idesc_hi : idesc_lo,
                                tmem + C::kTmemSfa + 4 * c, tmem + C::kTmemSfb + c * (BN / 32),
                                (kb | j) != 0 ? 1u : 0u);
                }
                tc_commit(&empty_bar[s]);
            }
            tc_commit(&accum_bar);  // the accumulator is final once every MMA above completed
            // TMEM is released at the end: make sure no MMA of this thread is still running then
            mbar_wait(&accum_bar, 0, kDrainLimitNs);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;                        // TMEM lanes this warp may read
        const int r = quarter * 32 + lane;
        const bool ready = mbar_wait(&accum_bar, 0, limit);
        tc_fence_after();
        const int64_t row = row0 + r;
        const bool live = ready && !mma_failed && row < row_end;
        const int64_t col0 = static_cast<int64_t>(n_tile) * BN;
#pragma unroll 1
        for (int cb = 0; cb < BN / 32; ++cb) {
            uint32_t v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + cb * 32, v);
            tmem_ld_wait();
            if (!live) continue;
            if (g.out_f32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(g.y) + row * g.N + col0 + cb * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(g.y) + row * g.N + col0 + cb * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t p[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 2 * k]),
                                                                  __uint_as_float(v[8 * i + 2 * k + 1]));
                        p[k] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    dst[i] = make_uint4(p[0], p[1], p[2], p[3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace macaq
