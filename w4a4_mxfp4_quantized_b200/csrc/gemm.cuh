// gemm.cuh -- block-scaled W4A4 GEMM on the sm_100a tensor cores (tcgen05.mma kind::mxf4).
//
//   Y[m, n] = sum_k (qa[m,k] * 2^(ea[m,k/32]-127)) * (qw[n,k] * 2^(ew[n,k/32]-127))
//
// fp32 accumulation in tensor memory, bf16 (round-to-nearest-even) or fp32 output. Dense and grouped
// (MoE) forms; the grouped form maps each 128-row tile to its expert from the device-side offsets.
// gemm_mxf4_pair_kernel is the dense form on 2-SM pairs (cta_group::2, 256-row tiles).
// Source: glonce.com page on MACaQ, paragraph 5 (W4A4 dense and grouped matmul kernels).
//
// Persistent kernel: one CTA per SM walks output tiles of 128 x BN (BN = 256, or 128 when
// N % 256 != 0) in a grouped raster (bands of kRasterM row tiles) so that the operands of the tiles
// in flight stay in L2. Warp roles (320 threads):
//   warp 0      TMA producer: per K-block of 256 elements, the A tile (128 rows x 128 bytes) and the
//               B tile (BN rows x 128 bytes) with 128-byte swizzle via tensor maps, plus the matching
//               scale-factor tiles (already in the tcgen05 128x4 tiling) by plain bulk copies. It runs
//               ahead across tile boundaries, limited only by the stage ring.
//   warp 1      TMEM allocator and MMA issuer: waits until the epilogue has drained the accumulator,
//               then per K-block copies the scale factors into TMEM (tcgen05.cp 32x128b.warpx4),
//               issues 4 MMAs of 128 x BN x 64 and frees the stage with tcgen05.commit; a final commit
//               per tile signals the epilogue.
//   warps 2-9   epilogue: tcgen05.ld of the fp32 accumulator (each warp reads its 32-lane quarter
//               and one half of the columns); for bf16 output the values are pulled into registers
//               and the accumulator released before the global stores, so the next tile's MMAs
//               overlap the stores.
// Every wait is bounded; a timeout anywhere stops all roles of the CTA, lets its own copies and
// MMAs land, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include "groups.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "swiglu.cuh"

namespace macaq {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 FP4 elements per K-block
constexpr int kGemmThreads = 320;   // producer warp, MMA warp, 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr int kRasterM = 16;   // row tiles per raster band
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
    int32_t raster_m;          // 2-SM kernel: 256-row tiles per raster band (<= 0: kRasterM)
};

template <int BN>
__host__ __device__ constexpr size_t gemm_smem_bytes(int E) {
    return GemmCfg<BN>::kSmemBytes + 2 * sizeof(int32_t) * (E + 1);
}

// Bounded wait that also gives up as soon as another role of the CTA has failed.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
                                                   volatile int *abort) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            record_timeout();
            *abort = 1;
            return false;
        }
    }
}

// Tile index -> (row tile, column tile) in bands of `bm` row tiles, columns inner.
__device__ __forceinline__ void raster(uint32_t t, uint32_t m_tiles, uint32_t n_tiles, uint32_t bm, uint32_t &mt,
                                       uint32_t &nt) {
    const uint32_t band = t / (bm * n_tiles);
    const uint32_t first = band * bm;
    const uint32_t height = min(bm, m_tiles - first);
    const uint32_t r = t - band * bm * n_tiles;
    mt = first + r % height;
    nt = r / height;
}
__device__ __forceinline__ void raster(uint32_t t, uint32_t m_tiles, uint32_t n_tiles, uint32_t &mt, uint32_t &nt) {
    raster(t, m_tiles, n_tiles, kRasterM, mt, nt);
}

// Epilogue of one output tile for one epilogue warp. Warp w (2..9) reads TMEM lane quarter w % 4
// (rows quarter*32 .. +31 of the CTA's 128) and column half (w - 2) / 4 of the BN columns. For bf16
// output the warp's 32 x BN/2 block is pulled into registers and the accumulator released (one
// arrival per warp on accum_empty, possibly in the leader CTA of a pair) before the global stores,
// so the next tile's MMAs overlap them; fp32 output keeps TMEM until its stores are issued.
template <int BN>
__device__ __forceinline__ void epilogue_tile(uint32_t tmem, int warp, int lane, int64_t row0, int64_t row_end,
                                              int64_t col0, const GemmArgs &g, uint32_t accum_empty_addr) {
    constexpr int kCols = BN / 2;  // columns per warp
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * kCols;
    const int64_t row = row0 + quarter * 32 + lane;
    const bool live = row < row_end;
    const int64_t c0 = col0 + half * kCols;
    if (g.out_f32) {
#pragma unroll 1
        for (int cb = 0; cb < kCols / 64; ++cb) {
            uint32_t v[64];
            tmem_ld64(taddr + cb * 64, v);
            tmem_ld_wait();
            if (!live) continue;
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(g.y) + row * g.N + c0 + cb * 64);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(accum_empty_addr);
    } else {
        uint32_t packed[kCols / 2];
#pragma unroll
        for (int cb = 0; cb < kCols / 64; ++cb) {
            uint32_t v[64];
            tmem_ld64(taddr + cb * 64, v);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                packed[cb * 32 + k] = *reinterpret_cast<uint32_t *>(&b2);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(accum_empty_addr);
        if (live) {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(g.y) + row * g.N + c0);
#pragma unroll
            for (int i = 0; i < kCols / 8; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
    }
}

// Epilogue of the 2-SM kernel: this warp's 32 accumulator rows x 128 columns leave TMEM first (the
// MMA warp gets the columns back at once), then go to Y through a 4 KB staging buffer as TMA stores
// of 32 rows x 128 bytes, so every write reaches L2 as whole 128-byte lines. The buffer holds 128-byte
// rows with the 16-byte chunks of row r at chunk position (k ^ r % 8), the TMA 128-byte swizzle, which
// keeps the warp's shared-memory writes free of bank conflicts. Rows at or past M are clipped by the
// tensor map.
__device__ __forceinline__ void store_chunk_tma(const CUtensorMap *ymap, uint8_t *buf, int lane, const uint32_t *w,
                                                int32_t col, int32_t row) {
    if (lane == 0) bulk_wait_read();  // the buffer's previous store has been read out
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 8; ++k)
        *reinterpret_cast<uint4 *>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) =
            make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(ymap, buf, col, row);
        bulk_commit();
    }
}

// row_end: rows at or past it are not written (the grouped form's expert bound; dense calls pass a
// bound past every row and rely on the tensor map's clipping). A warp whose 32 rows all lie below it
// stores through TMA; a warp that straddles it stores its live rows with plain 16-byte stores.
__device__ __forceinline__ void epilogue_tile_pair(uint32_t tmem, int warp, int lane, int32_t row0, int32_t col0,
                                                   bool out_f32, const CUtensorMap *ymap, uint8_t *buf,
                                                   uint32_t accum_empty_addr, int64_t row_end, void *y, int32_t ldy) {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 128;
    const int32_t row = row0 + quarter * 32;
    const int32_t col = col0 + half * 128;
    const bool whole = static_cast<int64_t>(row) + 32 <= row_end;
    const bool live = static_cast<int64_t>(row) + lane < row_end;
    if (out_f32) {
        uint32_t v[128];
        tmem_ld64(taddr, *reinterpret_cast<uint32_t(*)[64]>(v));
        tmem_ld64(taddr + 64, *reinterpret_cast<uint32_t(*)[64]>(v + 64));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(accum_empty_addr);
        if (whole) {
#pragma unroll
            for (int c = 0; c < 4; ++c) store_chunk_tma(ymap, buf, lane, v + 32 * c, col + 32 * c, row);
        } else if (live) {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<float *>(y) + (static_cast<int64_t>(row) + lane) * ldy + col);
#pragma unroll
            for (int c = 0; c < 32; ++c) dst[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
    } else {
        uint32_t packed[64];
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
            uint32_t v[64];
            tmem_ld64(taddr + cb * 64, v);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                packed[cb * 32 + k] = *reinterpret_cast<uint32_t *>(&b2);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(accum_empty_addr);
        if (whole) {
#pragma unroll
            for (int c = 0; c < 2; ++c) store_chunk_tma(ymap, buf, lane, packed + 32 * c, col + 64 * c, row);
        } else if (live) {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(y) + (static_cast<int64_t>(row) + lane) * ldy + col);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
        }
    }
}

template <int BN, bool kGrouped>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_mxf4_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap, GemmArgs g) {
    using C = GemmCfg<BN>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[S];
    __shared__ uint64_t empty_bar[S];
    __shared__ uint64_t accum_full;   // MMA -> epilogue: the tile's accumulator is final
    __shared__ uint64_t accum_empty;  // epilogue -> MMA: the accumulator has been read out
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int failed;   // set by any role whose wait ran out

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + S * C::kABytes;
    uint8_t *sSfa = sB + S * C::kBBytes;
    uint8_t *sSfb = sSfa + S * C::kSfaBytes;
    int32_t *s_off = reinterpret_cast<int32_t *>(sSfb + S * C::kSfbBytes);
    int32_t *s_tb = s_off + (g.E + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    griddep_wait();  // the operands and Y may belong to the previous kernel in the stream
    load_group_layout(kGrouped ? g.offsets : nullptr, kGrouped ? g.E : 1, g.rows, s_off, s_tb);  // block-wide
    const uint32_t m_tiles = static_cast<uint32_t>(s_tb[kGrouped ? g.E : 1]);
    const uint32_t n_tiles = static_cast<uint32_t>(g.N / BN);
    const uint32_t num_tiles = m_tiles * n_tiles;
    if (blockIdx.x >= num_tiles) return;  // uniform across the CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accum_full, 1);
        mbar_init(&accum_empty, kEpiWarps);  // one arrival per epilogue warp
        failed = 0;
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
    griddep_launch_dependents();
    const uint32_t tmem = tmem_slot;

    const int K = g.K;
    const int kq = K / 128;                      // scale tiles per SF row tile
    const int num_kb = (K + 255) / 256;
    const uint64_t limit = g.wait_limit_ns;

    // Which rows a row tile covers: its expert, first row, row bound.
    auto tile_rows = [&](uint32_t mt, int &expert, int64_t &row0, int64_t &row_end) {
        if constexpr (kGrouped) {
            int lo = 0, hi = g.E;  // s_tb[lo] <= mt < s_tb[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (static_cast<uint32_t>(s_tb[mid]) <= mt) lo = mid;
                else hi = mid;
            }
            expert = lo;
            row0 = s_off[lo] + static_cast<int64_t>(mt - s_tb[lo]) * kBM;
            row_end = s_off[lo + 1];
        } else {
            expert = 0;
            row0 = static_cast<int64_t>(mt) * kBM;
            row_end = g.rows;
        }
        if (row_end > row0 + kBM) row_end = row0 + kBM;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer
            uint32_t j = 0;  // global K-block counter across tiles (stage = j % S)
            bool stop = false;
            for (uint32_t t = blockIdx.x; t < num_tiles && !stop; t += gridDim.x) {
                uint32_t mt, nt;
                raster(t, m_tiles, n_tiles, mt, nt);
                int expert;
                int64_t row0, row_end;
                tile_rows(mt, expert, row0, row_end);
                const uint8_t *asf = g.asf + static_cast<uint64_t>(mt) * kq * 512;
                const uint8_t *bsf = g.bsf + static_cast<uint64_t>(expert) * g.bsf_stride +
                                     static_cast<uint64_t>(nt) * (BN / 128) * kq * 512;
                const int32_t brow = expert * g.N + static_cast<int32_t>(nt) * BN;
                for (int kb = 0; kb < num_kb; ++kb, ++j) {
                    const int s = j % S;
                    if (j >= S && !mbar_wait_or_abort(&empty_bar[s], ((j / S) & 1) ^ 1, limit, &failed)) {
                        stop = true;
                        break;
                    }
                    const int kch = (K - kb * 256) >= 256 ? 2 : 1;  // 128-element scale chunks in this block
                    mbar_arrive_expect_tx(&full_bar[s], C::kABytes + C::kBBytes + kch * 512 * (1 + BN / 128));
                    tma_load_2d(sA + s * C::kABytes, &amap, &full_bar[s], kb * kBKBytes, static_cast<int32_t>(row0));
                    tma_load_2d(sB + s * C::kBBytes, &bmap, &full_bar[s], kb * kBKBytes, brow);
                    bulk_load(sSfa + s * C::kSfaBytes, asf + kb * 1024, kch * 512, &full_bar[s]);
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h)
                        bulk_load(sSfb + s * C::kSfbBytes + h * 1024, bsf + static_cast<uint64_t>(h) * kq * 512 + kb * 1024,
                                  kch * 512, &full_bar[s]);
                }
            }
            // let the copies this thread issued land before the CTA can exit
            for (uint32_t i = (j > S ? j - S : 0); i < j; ++i)
                if (!mbar_wait(&full_bar[i % S], (i / S) & 1, kDrainLimitNs)) break;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t idesc_lo = idesc_mxf4(BN, 0);  // scale bytes 0-1 of each TMEM column
            const uint32_t idesc_hi = idesc_mxf4(BN, 2);  // scale bytes 2-3
            uint32_t j = 0;
            uint32_t tiles_done = 0;
            bool stop = false;
            for (uint32_t t = blockIdx.x; t < num_tiles && !stop; t += gridDim.x, ++tiles_done) {
                // the epilogue must have read the previous tile's accumulator out of TMEM
                if (tiles_done > 0 && !mbar_wait_or_abort(&accum_empty, (tiles_done - 1) & 1, limit, &failed)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < num_kb; ++kb, ++j) {
                    const int s = j % S;
                    if (!mbar_wait_or_abort(&full_bar[s], (j / S) & 1, limit, &failed)) {
                        stop = true;
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
                    for (int q = 0; q < 2 * kch; ++q) {
                        const int c = q >> 1;
                        // K step q covers bytes [32q, 32q + 32) of every 128-byte row
                        tc_mma_mxf4(tmem, adesc + 2 * q, bdesc + 2 * q, (q & 1) ? idesc_hi : idesc_lo,
                                    tmem + C::kTmemSfa + 4 * c, tmem + C::kTmemSfb + c * (BN / 32),
                                    (kb | q) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty_bar[s]);
                }
                tc_commit(&accum_full);  // the accumulator is final once every MMA above completed
            }
            // TMEM is released at the end: make sure no MMA of this thread is still running then.
            // The last commit is this phase's; if the loop stopped before any commit of the current
            // tile, commit once more so that the wait below covers everything issued.
            if (stop) {
                tc_commit(&accum_full);
                ++tiles_done;
            }
            if (tiles_done > 0) mbar_wait(&accum_full, (tiles_done - 1) & 1, kDrainLimitNs);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const uint32_t empty_addr = smem_u32(&accum_empty);
        uint32_t tiles_done = 0;
        for (uint32_t t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tiles_done) {
            uint32_t mt, nt;
            raster(t, m_tiles, n_tiles, mt, nt);
            int expert;
            int64_t row0, row_end;
            tile_rows(mt, expert, row0, row_end);
            if (!mbar_wait_or_abort(&accum_full, tiles_done & 1, limit, &failed)) break;
            tc_fence_after();
            if (failed) break;
            epilogue_tile<BN>(tmem, warp, lane, row0, row_end, static_cast<int64_t>(nt) * BN, g, empty_addr);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// ============================================================================ 2-SM pairs
// Dense GEMM on clusters of two CTAs (cta_group::2): a pair computes a 256 x 256 output tile. CTA r
// of the pair loads its 128 rows of A and rows [128r, 128r + 128) of the tile's 256 rows of B; the
// even CTA (the leader) issues the 256 x 256 x 64 MMAs, which read A and B from both CTAs' shared
// memory and leave each CTA's 128 rows of the accumulator in its own TMEM. Each CTA moves A + B/2
// per K-block instead of A + B.
//
// Scale factors: the MMA reads them from TMEM, four-fold replicated over the lane quarters. Six
// 32x128b.warpx4 copies per K-block (each about as costly as a whole 4 KB copy, together longer
// than the K-block's MMAs) are replaced by three 128x256b copies, whose source must hold the four
// replicas. TMA builds that source directly: a 4-D view of the tiled SF buffer, (128 bytes, tile
// half h, 8-row group i, 128x4 tile c) with strides (h: next tile, i: 128 B, c: 512 B), turns one
// 1 KB box into one replica laid out as [i][h][128 B]; four boxes give the 4 KB source of one copy.
// This path needs K % 256 == 0 (the K-block's two 128x4 tiles sit next to each other).
//
// Synchronisation: all TMA loads of both CTAs complete on the leader's full barrier (the leader
// expects both CTAs' bytes); the leader's commit frees the stage in both CTAs (multicast); the
// per-tile accumulator signals go to both CTAs; every epilogue warp of both CTAs releases the
// accumulator on the leader's accum_empty barrier.
struct PairCfg {
    static constexpr int kStages = 4;
    static constexpr int kABytes = 128 * kBKBytes;      // this CTA's 128 rows of A
    static constexpr int kBBytes = 128 * kBKBytes;      // this CTA's half of the 256 B rows
    static constexpr int kSfxBytes = 12288;             // replicated SF: A 4 KB, then B 4 KB per chunk
    static constexpr int kStageBytes = kABytes + kBBytes + kSfxBytes;
    static constexpr int kEpiBytes = kEpiWarps * 4096;  // one 32 x 128-byte store buffer per epilogue warp
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes;
    static constexpr int kTmemSfa = 256;
    static constexpr int kTmemSfb = 264;
    static constexpr int kTmemCols = 512;
    static constexpr int kThreads = kGemmThreads + 32;  // + a second producer warp for the scale factors
};

// ---------------------------------------------------------------- in-kernel quantization of A
// The fused layer (bf16 X in) for large M: the 2-SM GEMM quantizes X itself, once per element, into
// the workspace (the same codes and scales macaq_act_quant writes) and reads A from there by TMA. The
// work is cut into units of 16 rows x one 256-wide K-block, ordered as the GEMM's raster consumes A
// (by raster band, then K-block, then row tile). The host picks a low band (about two rounds of
// tiles per band) so that the first tiles need only the first band's rows: its units are taken by
// the idle epilogue warps at once, and later bands are quantized while earlier tiles accumulate. The epilogue warps, idle while a tile
// accumulates, take units whenever their own accumulator is not ready (the first one by warp index,
// the rest from a global counter); each
// finished unit adds one to the ready count of its (row tile, K-block) and to that of its row tile.
// At the start of a tile the A and scale-factor producers read the row tile's count once: when it is
// complete they load every K-block without further checks, otherwise they wait (bounded) for each
// K-block's count to complete before loading it, reading the counts of several K-blocks per trip. A unit never waits
// for anything and a warp waits for its accumulator only once every unit has been handed out, so all
// units finish. The last CTA to leave zeroes the counts and counters again (the workspace's counter
// region is zero before and after the call). Source: aipolix.com page, paragraph 2 (the transform of
// every layer's activations at inference).
struct FusedA {
    const uint16_t *x;     // bf16 [M, K]
    const float *inv_s;    // [K] multipliers 1/s, or nullptr
    uint8_t *xq;           // [M, K/2] codes (workspace)
    uint8_t *xsf;          // tiled SF of M rows (workspace)
    int32_t *flags;        // [rt_count][kb_count] finished units per (row tile, K-block)
    int32_t *rt_done;      // [rt_count] finished units per row tile (all K-blocks)
    int32_t *next_unit;    // units handed out
    int32_t *exit_count;   // CTAs that have left
    int32_t rt_count;      // ceil(M / 128)
    int32_t kb_count;      // K / 256
    int32_t units;         // rt_count * kb_count * kFaUnitsPerBlock
    int32_t band_rt;       // 128-row tiles per raster band of the GEMM (2 x its band of 256-row tiles)
};
constexpr int kFaRows = 16;
constexpr int kFaUnitsPerBlock = 128 / kFaRows;

__device__ __forceinline__ void fa_decode(const FusedA &f, int u, int &rt, int &kb, int &sub) {
    const int full_bands = f.rt_count / f.band_rt;
    const int per_band = f.kb_count * f.band_rt * kFaUnitsPerBlock;
    int band, rem, rts;
    if (u < full_bands * per_band) {
        band = u / per_band;
        rem = u - band * per_band;
        rts = f.band_rt;
    } else {
        band = full_bands;
        rem = u - full_bands * per_band;
        rts = f.rt_count - full_bands * f.band_rt;
    }
    kb = rem / (rts * kFaUnitsPerBlock);
    const int r2 = rem - kb * rts * kFaUnitsPerBlock;
    rt = band * f.band_rt + r2 / kFaUnitsPerBlock;
    sub = r2 % kFaUnitsPerBlock;
}

// One unit by one warp: kFaRows / 4 steps of 4 rows x 8 groups (lane = row (lane / 8), group
// (lane % 8) of the K-block, so the b >= 64 shuffles pair neighbouring groups of one row), the
// arithmetic of macaq_act_quant; rows past M get no codes and zero scales (padding rows of the tiled
// SF). All steps' loads are issued before the first step's arithmetic: one trip to memory per unit.
template <int kB>
__device__ __forceinline__ void fa_quant_unit(const FusedA &f, int u, int64_t M, int K, int lane) {
    int rt, kb, sub;
    fa_decode(f, u, rt, kb, sub);
    const uint32_t gcol = static_cast<uint32_t>(kb) * 8 + (lane & 7);
    const uint32_t kq = static_cast<uint32_t>(K / 128);
    const int64_t rows_sf = (M + 127) / 128 * 128;
    const int64_t m0 = static_cast<int64_t>(rt) * 128 + sub * kFaRows + (lane >> 3);
    uint4 raw[kFaRows / 4][4];
#pragma unroll
    for (int step = 0; step < kFaRows / 4; ++step) {
        const int64_t m = m0 + step * 4;
        if (m < M) {
            load_group_global(f.x + m * K + gcol * 32, raw[step]);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) raw[step][i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    uint64_t mv[16];
    if (f.inv_s != nullptr) load_mul(f.inv_s + gcol * 32, mv);
#pragma unroll
    for (int step = 0; step < kFaRows / 4; ++step) {
        const int64_t m = m0 + step * 4;
        uint64_t p[16];
        unpack_bf16x32(raw[step], p);
        if (f.inv_s != nullptr) {
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], mv[i]);
        }
        uint4 packed;
        uint32_t E8;
        transform_quantize_group<kB, false>(p, packed, E8);
        if (m < M) *reinterpret_cast<uint4 *>(f.xq + m * (K / 2) + gcol * 16) = packed;
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, E8, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, E8, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, E8, 3);
        if ((lane & 3) == 0 && m < rows_sf)
            *reinterpret_cast<uint32_t *>(f.xsf + sf_offset(static_cast<uint32_t>(m), gcol, kq)) =
                E8 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
    // the codes and scales are read by TMA (the async proxy) in other CTAs: order this thread's
    // generic writes before the counts that publish them
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
        __threadfence();
        atomicAdd(f.flags + rt * f.kb_count + kb, 1);
        atomicAdd(f.rt_done + rt, 1);
    }
}

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t *p) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// True when every unit of row tile rt (all K-blocks) has finished; row tiles past M have no units.
// Then the async proxy may read all of the row tile's codes and scales.
__device__ __forceinline__ bool fa_row_tile_ready(const FusedA &f, int rt) {
    if (rt >= f.rt_count) return true;
    if (ld_acquire_gpu(f.rt_done + rt) < f.kb_count * kFaUnitsPerBlock) return false;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

// Bounded wait until K-block kb of row tile rt has all its units finished (row tiles past M have
// none). The counts of up to kFaPeek K-blocks from kb are read together (relaxed loads, then one
// acquire fence), so a run of finished K-blocks costs one trip to L2; returns the end of the run of
// finished K-blocks (> kb), or -1 when the wait ran out or another role failed. Then the async proxy
// may read those K-blocks.
constexpr int kFaPeek = 8;
__device__ __forceinline__ int fa_wait_ready(const FusedA &f, int rt, int kb, uint64_t limit_ns, volatile int *abort) {
    if (rt >= f.rt_count) return f.kb_count;
    const int32_t *cnt = f.flags + rt * f.kb_count;
    const int n = min(kFaPeek, f.kb_count - kb);
    uint64_t t0 = 0;
    while (true) {
        int32_t v[kFaPeek];
#pragma unroll
        for (int i = 0; i < kFaPeek; ++i)
            if (i < n) asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v[i]) : "l"(cnt + kb + i) : "memory");
        int run = 0;
#pragma unroll
        for (int i = 0; i < kFaPeek; ++i)
            if (i < n && run == i && v[i] >= kFaUnitsPerBlock) run = i + 1;
        if (run > 0) {
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return kb + run;
        }
        if (*abort) return -1;
        if (t0 == 0) t0 = global_timer_ns();
        else if (global_timer_ns() - t0 > limit_ns) {
            record_timeout();
            *abort = 1;
            return -1;
        }
        __nanosleep(64);
    }
}

// Fused SwiGLU epilogue (kSwiglu = the down projection's Hadamard block b > 0): instead of writing
// Y, each epilogue warp takes its 32 rows x (64 gate + 64 up columns) of the accumulator, which with
// the 64-row gate/up interleave of the weights are intermediate channels [128 nt + 64 half, + 64),
// and writes their SwiGLU, transformed and MXFP4-quantized (swiglu.cuh), as the down projection's A
// operand: codes [M, I/2] and tiled SF. The gate/up output never reaches memory.
template <int kB>
__device__ __forceinline__ void epilogue_tile_pair_swiglu(uint32_t tmem, int warp, int lane, int32_t row0, int32_t nt,
                                                          int64_t M, const SwigluOut &o, uint32_t accum_empty_addr) {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 128;
    uint32_t gv[64], uv[64];
    tmem_ld64(taddr, gv);
    tmem_ld64(taddr + 64, uv);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(accum_empty_addr);
    const int32_t c0 = nt * 128 + half * 64;
    uint4 codes[2];
    uint32_t E8[2];
    swiglu_quant64<kB>(gv, uv, o.inv_s == nullptr ? nullptr : o.inv_s + c0, codes, E8);
    store_swiglu64(o, static_cast<int64_t>(row0) + quarter * 32 + lane, M, c0, codes, E8);
}

template <int kSwiglu, int kFusedB = 0, bool kGrouped = false>
__global__ void __launch_bounds__(PairCfg::kThreads, 1)
gemm_mxf4_pair_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                      const __grid_constant__ CUtensorMap sfamap, const __grid_constant__ CUtensorMap sfbmap,
                      const __grid_constant__ CUtensorMap ymap, GemmArgs g, int sf_replica_boxes, SwigluOut so,
                      FusedA fa) {
    using C = PairCfg;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[S];
    __shared__ uint64_t empty_bar[S];
    __shared__ uint64_t accum_full;
    __shared__ uint64_t accum_empty;   // used in the leader: 16 arrivals (8 warps x 2 CTAs) per tile
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int failed;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + S * C::kABytes;
    uint8_t *sSfx = sB + S * C::kBBytes;
    uint8_t *sEpi = sSfx + S * C::kSfxBytes;
    // grouped form: the expert row offsets, the first 128-row tile of each expert and the first
    // 256-row pair tile of each expert (each [E + 1]), after the epilogue buffers
    int32_t *s_off = reinterpret_cast<int32_t *>(sEpi + C::kEpiBytes);
    int32_t *s_tb = s_off + (g.E + 1);
    int32_t *s_pb = s_tb + (g.E + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const uint32_t cluster = blockIdx.x >> 1;
    const uint32_t clusters = gridDim.x >> 1;
    // dense: the host launches at most num_tiles pairs; grouped: the tile count is read on the device
    uint32_t m_tiles = static_cast<uint32_t>((g.rows + 255) / 256);
    const uint32_t n_tiles = static_cast<uint32_t>(g.N / 256);
    uint32_t num_tiles = m_tiles * n_tiles;
    const uint32_t band_m = g.raster_m > 0 ? static_cast<uint32_t>(g.raster_m) : static_cast<uint32_t>(kRasterM);
    const int K = g.K;
    const int kq = K / 128;
    const int num_kb = K / 256;
    const uint64_t limit = g.wait_limit_ns;
    // The pair's tiles: cluster, cluster + clusters, ... (tile t, all K-blocks [0, num_kb)).
    auto segment = [&](uint32_t i, uint32_t &t, int &k0, int &k1) -> bool {
        t = cluster + i * clusters;
        k0 = 0;
        k1 = num_kb;
        return t < num_tiles;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accum_full, 1);
        mbar_init(&accum_empty, 2 * kEpiWarps);
        // (the leader's full barrier: one expect-tx arrival; both producer warps' copies complete it)
        failed = 0;
        fence_mbar_init();
        prefetch_tensor_map(&amap);
        prefetch_tensor_map(&bmap);
        prefetch_tensor_map(&sfamap);
        prefetch_tensor_map(&sfbmap);
        prefetch_tensor_map(&ymap);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA signal
    tc_fence_after();
    griddep_wait();  // the operands and Y may belong to the previous kernel in the stream
    griddep_launch_dependents();
    if constexpr (kGrouped) {
        // pair tiles: expert e has ceil(tiles_e / 2) of them; s_pb is their exclusive prefix. Both CTAs
        // of a pair read the same offsets, so they walk the same tiles.
        load_group_layout(g.offsets, g.E, g.rows, s_off, s_tb);   // contains __syncthreads
        if (warp == 0) {
            int32_t carry = 0;
            for (int base = 0; base <= g.E; base += 32) {
                const int e = base + lane;
                int32_t x = (e > 0 && e <= g.E) ? (s_tb[e] - s_tb[e - 1] + 1) / 2 : 0;   // pair tiles of expert e - 1
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int32_t y = __shfl_up_sync(0xffffffffu, x, d);
                    if (lane >= d) x += y;
                }
                if (e <= g.E) s_pb[e] = carry + x;
                carry += __shfl_sync(0xffffffffu, x, 31);
            }
        }
        __syncthreads();
        m_tiles = static_cast<uint32_t>(s_pb[g.E]);
        num_tiles = m_tiles * n_tiles;
    }
    // grouped: pair-row tile mt -> its expert, this CTA's 128-row tile inside the SF layout (rt), its
    // first row and the expert's row bound (row_end <= row0 when this half lies past the expert)
    auto pair_rows = [&](uint32_t mt, int &expert, int32_t &rt, int64_t &row0, int64_t &row_end) {
        int lo = 0, hi = g.E;   // s_pb[lo] <= mt < s_pb[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (static_cast<uint32_t>(s_pb[mid]) <= mt) lo = mid;
            else hi = mid;
        }
        expert = lo;
        const int32_t local = static_cast<int32_t>(mt - static_cast<uint32_t>(s_pb[lo])) * 2 + static_cast<int32_t>(rank);
        rt = s_tb[lo] + local;
        row0 = s_off[lo] + static_cast<int64_t>(local) * 128;
        row_end = min(static_cast<int64_t>(s_off[lo + 1]), row0 + 128);
    };
    const uint32_t tmem = tmem_slot;
    const uint32_t leader_failed_addr = map_to_rank(smem_u32(const_cast<int *>(&failed)), 0);

    if (warp == 0 || warp == 10) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producers (both CTAs)
            // warp 0: A and B (and the expect-tx of both CTAs' bytes); warp 10: the scale factors
            const bool sf = warp == 10;
            uint32_t j = 0;
            bool stop = false;
            uint32_t t;
            int k0, k1;
            for (uint32_t sgi = 0; !stop && segment(sgi, t, k0, k1); ++sgi) {
                uint32_t mt, nt;
                raster(t, m_tiles, n_tiles, band_m, mt, nt);
                int32_t arow = static_cast<int32_t>(mt * 256 + rank * 128);
                int32_t brow = static_cast<int32_t>(nt * 256 + rank * 128);
                int32_t a_tile = static_cast<int32_t>((mt * 2 + rank) * kq);   // first 128x4 tile of A's rows
                int32_t b_tile = static_cast<int32_t>(nt * 2 * kq);            // of B's first 128 rows
                if constexpr (kGrouped) {
                    // a half past its expert loads whatever rows and scales lie there (zeros past the
                    // tensors); the epilogue writes none of its rows
                    int expert, rt;
                    int64_t row0, row_end;
                    pair_rows(mt, expert, rt, row0, row_end);
                    arow = static_cast<int32_t>(row0);
                    a_tile = rt * kq;
                    brow = expert * g.N + static_cast<int32_t>(nt * 256 + rank * 128);
                    b_tile = (expert * (g.N / 128) + static_cast<int32_t>(nt * 2)) * kq;
                }
                // fused form: once the row tile's units have all finished, its K-blocks need no checks;
                // otherwise a_ready_end is the end of the run of K-blocks known to be finished
                int a_ready_end = num_kb;
                if constexpr (kFusedB > 0)
                    if (!fa_row_tile_ready(fa, static_cast<int>(mt * 2 + rank))) a_ready_end = 0;
                for (int kb = k0; kb < k1; ++kb, ++j) {
                    const int s = j % S;
                    if (j >= S && !mbar_wait_or_abort(&empty_bar[s], ((j / S) & 1) ^ 1, limit, &failed)) {
                        stop = true;
                        break;
                    }
                    if constexpr (kFusedB > 0) {   // A (codes or scales) of this K-block written in this launch
                        if (kb >= a_ready_end) {
                            a_ready_end = fa_wait_ready(fa, static_cast<int>(mt * 2 + rank), kb, limit, &failed);
                            if (a_ready_end < 0) {
                                stop = true;
                                break;
                            }
                        }
                    }
                    if (!sf) {
                        if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * C::kStageBytes);
                        tma_load_2d_pair(sA + s * C::kABytes, &amap, &full_bar[s], kb * kBKBytes, arow);
                        tma_load_2d_pair(sB + s * C::kBBytes, &bmap, &full_bar[s], kb * kBKBytes, brow);
                    } else {
                        // four replicas each: A (halves = the K-block's tiles), B chunk 0, 1 (halves = rows)
                        uint8_t *x = sSfx + s * C::kSfxBytes;
                        if (sf_replica_boxes == 1) {
                            tma_load_5d_pair(x, &sfamap, &full_bar[s], 0, 0, 0, 0, a_tile + 2 * kb);
                            tma_load_5d_pair(x + 4096, &sfbmap, &full_bar[s], 0, 0, 0, 0, b_tile + 2 * kb);
                            tma_load_5d_pair(x + 8192, &sfbmap, &full_bar[s], 0, 0, 0, 0, b_tile + 2 * kb + 1);
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                tma_load_4d_pair(x + q * 1024, &sfamap, &full_bar[s], 0, 0, 0, a_tile + 2 * kb);
                                tma_load_4d_pair(x + 4096 + q * 1024, &sfbmap, &full_bar[s], 0, 0, 0, b_tile + 2 * kb);
                                tma_load_4d_pair(x + 8192 + q * 1024, &sfbmap, &full_bar[s], 0, 0, 0, b_tile + 2 * kb + 1);
                            }
                        }
                    }
                }
            }
            // the leader's full barriers count both CTAs' bytes: let every issued copy land
            if (leader && !sf)
                for (uint32_t i = (j > S ? j - S : 0); i < j; ++i)
                    if (!mbar_wait(&full_bar[i % S], (i / S) & 1, kDrainLimitNs)) break;
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------------------ MMA issuer (leader only)
            const uint32_t idesc_lo = idesc_mxf4_m(256, 256, 0);
            const uint32_t idesc_hi = idesc_mxf4_m(256, 256, 2);
            uint32_t j = 0;
            uint32_t tiles_done = 0;
            bool stop = false;
            uint32_t t;
            int k0, k1;
            for (uint32_t sgi = 0; !stop && segment(sgi, t, k0, k1); ++sgi, ++tiles_done) {
                if (tiles_done > 0 && !mbar_wait_or_abort(&accum_empty, (tiles_done - 1) & 1, limit, &failed)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                for (int kb = k0; kb < k1; ++kb, ++j) {
                    const int s = j % S;
                    if (!mbar_wait_or_abort(&full_bar[s], (j / S) & 1, limit, &failed)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfx = smem_u32(sSfx + s * C::kSfxBytes);
                    tc_cp_sf_wide_pair(tmem + C::kTmemSfa, sdesc_sf_wide(sfx));
                    tc_cp_sf_wide_pair(tmem + C::kTmemSfb, sdesc_sf_wide(sfx + 4096));
                    tc_cp_sf_wide_pair(tmem + C::kTmemSfb + 8, sdesc_sf_wide(sfx + 8192));
                    const uint64_t adesc = sdesc_sw128(smem_u32(sA + s * C::kABytes));
                    const uint64_t bdesc = sdesc_sw128(smem_u32(sB + s * C::kBBytes));
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c = q >> 1;
                        tc_mma_mxf4_pair(tmem, adesc + 2 * q, bdesc + 2 * q, (q & 1) ? idesc_hi : idesc_lo,
                                         tmem + C::kTmemSfa + 4 * c, tmem + C::kTmemSfb + c * 8, (kb != k0 || q != 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&empty_bar[s]);
                }
                tc_commit_pair(&accum_full);
            }
            if (stop) {
                tc_commit_pair(&accum_full);
                ++tiles_done;
            }
            if (tiles_done > 0) mbar_wait(&accum_full, (tiles_done - 1) & 1, kDrainLimitNs);
        }
    } else if (warp >= 2 && warp < 10) {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const uint32_t empty_addr = map_to_rank(smem_u32(&accum_empty), 0);
        uint32_t tiles_done = 0;
        uint32_t t;
        int k0, k1;
        bool units_left = kFusedB > 0;
        // one unit of A's quantization (fused form), unless every unit has been handed out. Epilogue
        // warp w of the launch takes unit w first (all of them start idle, so no counter is needed);
        // later units come from the shared counter, past the first gridDim.x * kEpiWarps
        const int first_unit = static_cast<int>(blockIdx.x) * kEpiWarps + (warp - 2);
        bool took_first = false;
        auto take_unit = [&]() {
            if constexpr (kFusedB > 0) {
                int u = first_unit;
                if (took_first) {
                    if (lane == 0) u = static_cast<int>(gridDim.x) * kEpiWarps + atomicAdd(fa.next_unit, 1);
                    u = __shfl_sync(0xffffffffu, u, 0);
                }
                took_first = true;
                if (u >= fa.units) {
                    units_left = false;
                    return;
                }
                fa_quant_unit<kFusedB>(fa, u, g.rows, g.K, lane);
            }
        };
        for (uint32_t sgi = 0; segment(sgi, t, k0, k1); ++sgi, ++tiles_done) {
            uint32_t mt, nt;
            raster(t, m_tiles, n_tiles, band_m, mt, nt);
            int64_t row0 = static_cast<int64_t>(mt) * 256 + rank * 128, row_end = int64_t(1) << 62;   // dense: TMA clips at M
            if constexpr (kGrouped) {
                int expert, rt;
                pair_rows(mt, expert, rt, row0, row_end);
            }
            if constexpr (kFusedB > 0) {
                // test_wait, not try_wait: a blocking poll would hold the warp for the suspend limit
                // between units while the accumulator is far from ready
                while (units_left && !failed && !mbar_test_wait(smem_u32(&accum_full), tiles_done & 1)) take_unit();
            }
            if (!mbar_wait_or_abort(&accum_full, tiles_done & 1, limit, &failed)) break;
            tc_fence_after();
            int leader_failed;
            asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(leader_failed) : "r"(leader_failed_addr) : "memory");
            if (failed || leader_failed) break;
            if constexpr (kSwiglu > 0)
                epilogue_tile_pair_swiglu<kSwiglu>(tmem, warp, lane, static_cast<int32_t>(mt * 256 + rank * 128),
                                                   static_cast<int32_t>(nt), g.rows, so, empty_addr);
            else
                epilogue_tile_pair(tmem, warp, lane, static_cast<int32_t>(row0), static_cast<int32_t>(nt * 256),
                                   g.out_f32 != 0, &ymap, sEpi + (warp - 2) * 4096, empty_addr, row_end, g.y, g.N);
        }
        while (units_left && !failed) take_unit();   // units other pairs still wait for
        if (lane == 0) bulk_wait_read();  // shared memory stays valid until this warp's stores have read it
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its partner may still touch its barriers or shared memory
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, C::kTmemCols);
    if constexpr (kFusedB > 0) {
        // the last CTA to leave (every other CTA has finished its units and its waits) zeroes the
        // ready counts and counters for the workspace's next use
        __shared__ int s_last_cta;
        if (threadIdx.x == 0) {
            __threadfence();
            s_last_cta = atomicAdd(fa.exit_count, 1) == static_cast<int>(gridDim.x) - 1;
        }
        __syncthreads();
        if (s_last_cta) {
            __threadfence();
            for (int i = threadIdx.x; i < fa.rt_count * fa.kb_count; i += blockDim.x) fa.flags[i] = 0;
            for (int i = threadIdx.x; i < fa.rt_count; i += blockDim.x) fa.rt_done[i] = 0;
            if (threadIdx.x == 0) {
                *fa.next_unit = 0;
                *fa.exit_count = 0;
            }
        }
    }
}

// ============================================================================ skinny (small M)
// Dense GEMM for few rows (M <= 128, e.g. decode): the layer is a stream over W', so the weights take
// the MMA's 128-row M slot and the M activation rows (padded to Mp, a multiple of 16) take its N
// slot: D^T[n, m] = sum_k W'[n, k] X'[m, k]. The flattened space of (128-row W tile, K-block) units is
// cut into equal contiguous ranges, one per CTA (one CTA per SM), so every SM streams the same number
// of bytes. A CTA's range covers pieces of one or more tiles; a tile covered by one CTA is written
// straight to Y (bf16 through shared memory and a TMA store), otherwise each piece's fp32 partial goes
// to the workspace and the CTA that completes the tile's last piece (an atomic count per tile) adds
// the pieces in their fixed order, writes Y and sets the count back to zero. The counters live in the
// workspace's first 64 KiB, which is therefore zero between calls whatever the shapes of earlier
// calls; the partials behind them are written before they are read. When splitting tiles
// would move more partial bytes than it saves (large M), the ranges are cut on whole tiles instead.
// Both operands' scale factors arrive replicated (zero-stride TMA view) and go to TMEM with one wide
// 128x256b copy each per K-block. The stage ring has up to kSkinnyMaxStages stages; the accumulator
// is double-buffered in TMEM. Needs K % 256 == 0.
//
// Fused form (kFusedB = Hadamard block b > 0; dispatched, and tested, for M <= kSkinnyFusedMaxM = 4
// only, where it is faster than a separate quantizer launch; the host also requires a stage count
// divisible by four, so each quantizer warp owns whole stages): the activations arrive as bf16 X. Per stage
// the producer also loads X's K-block (16 rows x 256 bf16 by TMA, zero-filled past M) and the
// K-block's 256 multipliers 1/s (bulk copy); four quantizer warps (warps 6-9, one 32-element group
// per thread: row t / 8, group t % 8) apply scale, Hadamard and MXFP4 exactly as the quantizer kernel
// does, and write the codes (128-byte swizzled, as the MMA's descriptor reads them) and the E8M0
// exponents (four-fold replicated, as the wide copy reads them) straight into the stage. No quantized
// activation ever goes to HBM. Source: the aipolix.com page, paragraph 2 (transform on each layer's
// activations at inference); glonce.com page, paragraph 5 (W4A4 dense matmul).
constexpr int kSkinnyMaxStages = 4;   // deeper rings measured slower on the decode shapes
constexpr int kSkinnyFusedMaxM = 4;

struct SkinnyArgs {
    void *y;                   // [M, N]
    float *partials;           // [tiles][max_pieces][M][128] fp32, written before read
    int32_t *counts;           // [tiles], zero between calls (the workspace's first 64 KiB)
    int32_t M, N, K;
    int32_t mp;                // M rounded up to 16: the MMA's N
    int32_t out_f32;
    int32_t stages;
    int32_t max_pieces;
    uint32_t units;            // (N / 128) * (K / 256)
    uint32_t gran;             // units per indivisible chunk: 1 (split tiles) or K-blocks per tile (whole tiles)
    uint64_t wait_limit_ns;
    const float *inv_s;        // fused form: [K] multipliers 1/s, or nullptr for s = 1
};

__host__ __device__ constexpr int skinny_stage_bytes(int mp) { return 128 * kBKBytes + mp * kBKBytes + 8192; }
// fused form: + the K-block of bf16 X (mp rows x 512 bytes) and of the multipliers (1 KB)
__host__ __device__ constexpr int skinny_stage_bytes_fused(int mp) { return skinny_stage_bytes(mp) + mp * 512 + 1024; }
__host__ __device__ constexpr int skinny_stage_bytes_y(int mp) { return mp * 128 * 2; }  // bf16 staging of one tile

// Epilogue of the skinny kernels (warps 2-5, one TMEM lane quarter each): for every piece of a weight
// tile this CTA covers, wait for its accumulator (buffer b = piece parity at tmem + 128 b), then either
// write Y (a tile covered by one CTA: bf16 staged in shared memory and stored by TMA, or fp32 direct)
// or publish the piece's fp32 partial and, in the CTA that completes the tile, add the pieces in their
// fixed order and write Y. The CTA covering unit u is the largest c with floor(c * chunks / C) <= u /
// gran, C = gridDim.x.
__device__ __forceinline__ void skinny_epilogue(const SkinnyArgs &g, const CUtensorMap *ymap, uint32_t tmem, int warp, int lane,
                                                uint8_t *sY, int mp, uint64_t *accum_full, uint64_t *accum_empty,
                                                volatile int *failed, int32_t *s_last, uint64_t limit, uint32_t u_begin,
                                                uint32_t u_end, uint32_t num_kb, uint32_t chunks) {
    const uint32_t C = gridDim.x;
    auto cta_of = [&](uint32_t u) {
        return static_cast<uint32_t>(((static_cast<uint64_t>(u / g.gran) + 1) * C - 1) / chunks);
    };
    const int quarter = warp & 3;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int nl = quarter * 32 + lane;          // W row inside the tile
    uint8_t *ystage = sY + static_cast<size_t>(quarter) * mp * 64;  // [mp][32] bf16 of this warp
    uint32_t piece = 0;
    for (uint32_t u = u_begin; u < u_end; ++piece) {
        const uint32_t tile = u / num_kb;
        const uint32_t u_first = tile * num_kb;
        const uint32_t u_stop = min(u_end, u_first + num_kb);
        const uint32_t c_first = cta_of(u_first), c_last = cta_of(u_first + num_kb - 1);
        const int npieces = static_cast<int>(c_last - c_first + 1);
        const int pidx = static_cast<int>(blockIdx.x - c_first);
        u = u_stop;
        const int b = piece & 1;
        bool ok = mbar_wait_or_abort(&accum_full[b], (piece >> 1) & 1, limit, failed);
        tc_fence_after();
        // the four epilogue warps meet at named barriers below (split tiles): they stop together
        // or not at all, so a wait that ran out in one warp never leaves the others at a barrier
        if (!bar_and(1, 128, ok && !*failed)) break;
        const int64_t n = static_cast<int64_t>(tile) * 128 + nl;
        const bool staged = npieces == 1 && !g.out_f32;
        if (staged) {  // the previous tile's store (issued by lane 0) has read the staging buffer
            if (lane == 0) bulk_wait_read();
            __syncwarp();
        }
        float *part = g.partials + ((static_cast<uint64_t>(tile) * g.max_pieces + pidx) * g.M) * 128;
        auto emit = [&](int m0, const uint32_t (&v)[32]) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int m = m0 + i;
                const float f = __uint_as_float(v[i]);
                if (staged) {
                    if (m < mp) reinterpret_cast<__nv_bfloat16 *>(ystage)[m * 32 + lane] = __float2bfloat16_rn(f);
                } else if (m < g.M) {
                    if (npieces == 1) static_cast<float *>(g.y)[static_cast<int64_t>(m) * g.N + n] = f;
                    else __stcg(part + static_cast<int64_t>(m) * 128 + nl, f);
                }
            }
        };
        for (int m0 = 0; m0 < mp; m0 += 64) {  // two TMEM loads in flight per wait
            uint32_t v0[32], v1[32];
            tmem_ld32(taddr + 128 * b + m0, v0);
            if (m0 + 32 < mp) tmem_ld32(taddr + 128 * b + m0 + 32, v1);
            tmem_ld_wait();
            emit(m0, v0);
            if (m0 + 32 < mp) emit(m0 + 32, v1);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accum_empty[b]);
        if (staged) {
            fence_proxy_async_smem();  // generic writes -> the TMA store's reads
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(ymap, ystage, static_cast<int32_t>(tile * 128 + quarter * 32), 0);
                bulk_commit();
            }
        }
        if (npieces > 1) {
            // publish this piece, then let the CTA that completes the tile add the pieces in order.
            // The barrier orders every thread's partial stores before thread 0's fence and count
            // increment (a cumulative release); the reader side mirrors it.
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (warp == 2 && lane == 0) {
                __threadfence();
                *s_last = atomicAdd(&g.counts[tile], 1) == npieces - 1;
                __threadfence();
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (*s_last) {
                // the pieces are added in their fixed order (piece 0 first); four pieces x 16 rows of
                // loads are in flight per round trip to L2
                float *base = g.partials + (static_cast<uint64_t>(tile) * g.max_pieces) * g.M * 128 + nl;
                for (int m0 = 0; m0 < g.M; m0 += 16) {
                    float acc[16];
                    for (int p0 = 0; p0 < npieces; p0 += 4) {
                        float v[4][16];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                v[q][i] = (p0 + q < npieces && m0 + i < g.M)
                                              ? __ldcg(base + (static_cast<uint64_t>(p0 + q) * g.M + m0 + i) * 128)
                                              : 0.0f;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (p0 + q >= npieces) break;
#pragma unroll
                            for (int i = 0; i < 16; ++i) acc[i] = (p0 + q == 0) ? v[q][i] : acc[i] + v[q][i];
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int m = m0 + i;
                        if (m >= g.M) break;
                        if (g.out_f32) static_cast<float *>(g.y)[static_cast<int64_t>(m) * g.N + n] = acc[i];
                        else static_cast<__nv_bfloat16 *>(g.y)[static_cast<int64_t>(m) * g.N + n] = __float2bfloat16_rn(acc[i]);
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (warp == 2 && lane == 0) g.counts[tile] = 0;  // ready for the next call
            }
        }
    }
    if (lane == 0) bulk_wait_read();  // shared memory stays valid until this warp's stores have read it
}

template <int kFusedB>
__global__ void __launch_bounds__(kFusedB > 0 ? 320 : 192, 1)
gemm_mxf4_skinny_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                        const __grid_constant__ CUtensorMap sfwmap, const __grid_constant__ CUtensorMap sfxmap,
                        const __grid_constant__ CUtensorMap ymap, SkinnyArgs g) {
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[kSkinnyMaxStages];
    __shared__ uint64_t empty_bar[kSkinnyMaxStages];
    __shared__ uint64_t xin_bar[kSkinnyMaxStages];   // fused form: X and 1/s of the stage have landed
    __shared__ uint64_t accum_full[2];
    __shared__ uint64_t accum_empty[2];
    __shared__ uint64_t mma_done;
    __shared__ uint32_t tmem_slot;
    __shared__ int32_t s_last;
    __shared__ volatile int failed;

    constexpr bool kFused = kFusedB > 0;
    const int S = g.stages;
    const int mp = g.mp;
    const int stage_bytes = kFused ? skinny_stage_bytes_fused(mp) : skinny_stage_bytes(mp);
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint8_t *sY = smem + S * stage_bytes;  // [4 warps][mp rows][32 columns] bf16
    auto sW = [&](int s) { return smem + s * stage_bytes; };
    auto sX = [&](int s) { return smem + s * stage_bytes + 128 * kBKBytes; };
    auto sSfw = [&](int s) { return smem + s * stage_bytes + (128 + mp) * kBKBytes; };
    auto sSfx = [&](int s) { return smem + s * stage_bytes + (128 + mp) * kBKBytes + 4096; };
    auto sXin = [&](int s) { return smem + s * stage_bytes + skinny_stage_bytes(mp); };
    auto sInv = [&](int s) { return smem + s * stage_bytes + skinny_stage_bytes(mp) + mp * 512; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = g.K;
    const int kq = K / 128;
    const uint32_t num_kb = static_cast<uint32_t>(K / 256);
    const uint32_t C = gridDim.x;
    const uint32_t chunks = g.units / g.gran;  // ranges are cut on chunk boundaries
    const uint32_t u_begin = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x) * chunks) / C) * g.gran;
    const uint32_t u_end = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x + 1) * chunks) / C) * g.gran;
    const uint64_t limit = g.wait_limit_ns;

    // The weights do not depend on the previous kernel in the stream, and their loads need only this
    // CTA's barriers: thread 0 requests the first stages' W' tiles and scale factors right after it
    // has initialised the barriers, before TMEM is allocated (which may wait for the previous
    // kernel's CTA on this SM to free its columns) and before the CTA-wide barrier.
    auto load_w = [&](uint32_t u, int s) {
        const uint32_t tile = u / num_kb;
        const int kb = static_cast<int>(u - tile * num_kb);
        if constexpr (kFused) mbar_arrive_expect_tx(&full_bar[s], 128 * kBKBytes + 4096);
        else mbar_arrive_expect_tx(&full_bar[s], (128 + mp) * kBKBytes + 8192);
        tma_load_2d(sW(s), &wmap, &full_bar[s], kb * kBKBytes, static_cast<int32_t>(tile * 128));
        tma_load_5d(sSfw(s), &sfwmap, &full_bar[s], 0, 0, 0, 0, static_cast<int32_t>(tile * kq + 2 * kb));
    };
    const uint32_t pre = min(static_cast<uint32_t>(S), u_end > u_begin ? u_end - u_begin : 0u);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], kFused ? 2 : 1);   // fused: the producer and the stage's quantizer warp
            mbar_init(&empty_bar[s], 1);
            mbar_init(&xin_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accum_full[b], 1);
            mbar_init(&accum_empty[b], 4);
        }
        mbar_init(&mma_done, 1);
        failed = 0;
        fence_mbar_init();
        prefetch_tensor_map(&wmap);
        prefetch_tensor_map(&sfwmap);
        for (uint32_t i = 0; i < pre; ++i) load_w(u_begin + i, static_cast<int>(i));
        prefetch_tensor_map(&xmap);
        prefetch_tensor_map(&sfxmap);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    if constexpr (kFused) {
        // the quantizer writes only the codes and scale bytes of rows < M; the rest of the X operand
        // and of each replicated scale block stays zero for the whole launch
        for (int s = 0; s < S; ++s) {
            for (int i = threadIdx.x; i < 4096 / 16; i += blockDim.x)
                reinterpret_cast<uint4 *>(sSfx(s))[i] = make_uint4(0u, 0u, 0u, 0u);
            for (int i = threadIdx.x; i < mp * kBKBytes / 16; i += blockDim.x)
                reinterpret_cast<uint4 *>(sX(s))[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch_dependents();
    const uint32_t tmem = tmem_slot;                 // accumulators at columns 0 and 128
    const uint32_t t_sfw = tmem + 256, t_sfx = tmem + 264;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer
            // The first `pre` stages' weights were requested at set-up; the activations may belong to
            // the previous kernel, so they are requested after waiting for it.
            auto load_x = [&](uint32_t u, int s) {
                const int kb = static_cast<int>(u % num_kb);
                if constexpr (kFused) {
                    // X's K-block as bf16 (rows past M read as zero) and its 256 multipliers
                    mbar_arrive_expect_tx(&xin_bar[s], mp * 512 + (g.inv_s != nullptr ? 1024 : 0));
                    tma_load_2d(sXin(s), &xmap, &xin_bar[s], kb * 256, 0);
                    if (g.inv_s != nullptr) bulk_load(sInv(s), g.inv_s + kb * 256, 1024, &xin_bar[s]);
                } else {
                    tma_load_2d(sX(s), &xmap, &full_bar[s], kb * kBKBytes, 0);
                    tma_load_5d(sSfx(s), &sfxmap, &full_bar[s], 0, 0, 0, 0, 2 * kb);
                }
            };
            griddep_wait();
            for (uint32_t i = 0; i < pre; ++i) load_x(u_begin + i, static_cast<int>(i));
            uint32_t j = pre;
            for (uint32_t u = u_begin + pre; u < u_end; ++u, ++j) {
                const int s = j % S;
                if (!mbar_wait_or_abort(&empty_bar[s], ((j / S) & 1) ^ 1, limit, &failed)) break;
                load_w(u, s);
                load_x(u, s);
            }
            for (uint32_t i = (j > static_cast<uint32_t>(S) ? j - S : 0); i < j; ++i)
                if (!mbar_wait(&full_bar[i % S], (i / S) & 1, kDrainLimitNs)) break;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t idesc_lo = idesc_mxf4(mp, 0), idesc_hi = idesc_mxf4(mp, 2);
            uint32_t j = 0, piece = 0;
            bool stop = false;
            for (uint32_t u = u_begin; u < u_end && !stop; ++piece) {
                const uint32_t tile = u / num_kb;
                const uint32_t u_stop = min(u_end, (tile + 1) * num_kb);
                const int b = piece & 1;
                if (piece >= 2 && !mbar_wait_or_abort(&accum_empty[b], ((piece >> 1) - 1) & 1, limit, &failed)) break;
                tc_fence_after();
                for (bool first = true; u < u_stop; ++u, ++j, first = false) {
                    const int s = j % S;
                    if (!mbar_wait_or_abort(&full_bar[s], (j / S) & 1, limit, &failed)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    tc_cp_sf_wide(t_sfw, sdesc_sf_wide(smem_u32(sSfw(s))));
                    tc_cp_sf_wide(t_sfx, sdesc_sf_wide(smem_u32(sSfx(s))));
                    const uint64_t wdesc = sdesc_sw128(smem_u32(sW(s)));
                    const uint64_t xdesc = sdesc_sw128(smem_u32(sX(s)));
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c = q >> 1;
                        tc_mma_mxf4(tmem + 128 * b, wdesc + 2 * q, xdesc + 2 * q, (q & 1) ? idesc_hi : idesc_lo,
                                    t_sfw + 4 * c, t_sfx + 4 * c, (first && q == 0) ? 0u : 1u);
                    }
                    tc_commit(&empty_bar[s]);
                }
                tc_commit(&accum_full[b]);
            }
            // every MMA issued must be done before TMEM is released
            tc_commit(&mma_done);
            mbar_wait(&mma_done, 0, kDrainLimitNs);
        }
    } else if (kFused && warp >= 6) {
        // ---------------------------------------------------------------- quantizer (fused form)
        // Warp 6 + w takes the stages j = w, w + 4, ...: four K-blocks are quantized at once. In a
        // K-block, group index gi = 8 row + (32-element group); lane l takes gi = l, l + 32, ... over
        // the M live rows (adjacent lanes hold adjacent groups of one row, as the b >= 64 shuffles
        // need). Rows M..15 were zeroed once and stay zero.
        const int qw = warp - 6;
        const int live = g.M * 8;
        uint32_t j = qw;
        for (uint32_t u = u_begin + qw; u < u_end; u += 4, j += 4) {
            const int s = j % S;
            // the whole warp leaves together if any lane's wait ran out (the Hadamard may shuffle)
            if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&xin_bar[s], (j / S) & 1, limit, &failed))) break;
            for (int gi0 = 0; gi0 < live; gi0 += 32) {
                const int gi = gi0 + lane;
                const int m = gi >> 3;           // row
                const int gq = gi & 7;           // 32-element group inside the K-block
                uint4 raw[4] = {};
                if (gi < live) {
                    const uint8_t *src = sXin(s) + m * 512 + gq * 64;
#pragma unroll
                    for (int i = 0; i < 4; ++i) raw[i] = *reinterpret_cast<const uint4 *>(src + i * 16);
                }
                uint64_t p[16];
                unpack_bf16x32(raw, p);
                if (g.inv_s != nullptr) {
                    const float4 *mv4 = reinterpret_cast<const float4 *>(sInv(s) + gq * 128);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 f = mv4[i];
                        p[2 * i] = mul2(p[2 * i], pk2(f.x, f.y));
                        p[2 * i + 1] = mul2(p[2 * i + 1], pk2(f.z, f.w));
                    }
                }
                uint4 packed;
                uint32_t E8;
                transform_quantize_group<kFusedB, false>(p, packed, E8);
                if (gi < live) {
                    // codes: row m's 16-byte chunk gq of the 128-byte row, 128-byte swizzle
                    *reinterpret_cast<uint4 *>(sX(s) + m * 128 + ((gq ^ (m & 7)) << 4)) = packed;
                    // exponent: SF tile half gq / 4, column gq % 4, row m (lane m of 32, row quarter 0),
                    // in each of the four replicas (1 KB apart)
                    uint8_t *sf = sSfx(s) + ((m >> 3) * 2 + (gq >> 2)) * 128 + (m & 7) * 16 + (gq & 3);
#pragma unroll
                    for (int q = 0; q < 4; ++q) sf[q * 1024] = static_cast<uint8_t>(E8);
                }
            }
            // the stage's input has been read and its operands written: order both before the MMA's
            // (async-proxy) reads and the next TMA write of the stage
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_bar[s]);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-5)
        skinny_epilogue(g, &ymap, tmem, warp, lane, sY, mp, accum_full, accum_empty, &failed, &s_last, limit, u_begin,
                        u_end, num_kb, chunks);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace macaq
