// w4a16.cuh -- weight-only mode: MXFP4 weights W' x bf16 activations, for decode (M <= 64).
//
// Page "MACaQ quantizer from huawei-csl targets GGUF, vLLM and Diffusers models" (glonce.com),
// paragraph 3: the vLLM backend serves W4A4 or weight-only checkpoints. In the weight-only mode the
// weights are the same prepared W' = MXFP4(W diag(s) H_b / b), and the activations get the same
// online transform X' = X diag(1/s) H_b in fp32 (macaq_act_transform, the act_quant arithmetic without
// the MXFP4 step) but stay unquantized: rounded once to bf16, the tensor cores' operand type. So
//     Y[m, n] = sum_k bf16(X'[m, k]) * dq(W'[n, k]),   fp32 accumulation.
//
// B200 mapping: the skinny swap-AB plan (W' tiles of 128 rows in the MMA's M slot, the M <= 64 rows
// of X' in its N slot, the (tile, K-block) units split evenly over the SMs, split tiles reduced
// through the workspace). Per 256-wide K-block the producer TMA-loads W's codes (128 rows x 128 B,
// 128-byte swizzle), their 1 KB of scale factors and X' (four 64-column bf16 atoms, 128-byte swizzle:
// the MMA's B operand as is). Four dequant warps expand the codes: a table of the 256 code bytes'
// two unscaled values as bf16x2 (one copy per shared-memory bank, so every lane reads its own copy),
// times the group's power-of-two scale with one bf16x2 multiply (exact for scales E8M0 <= 252), and
// write the 128 x 256 bf16 operand straight into tensor memory (tcgen05.st, one lane per weight
// row). tcgen05.mma kind::f16 reads A from tensor memory and B from shared memory. Two A buffers in
// TMEM let the dequant warps fill one K-block while the MMAs read the other.
#pragma once

#include "gemm.cuh"

namespace macaq {

constexpr int kWoMaxStages = 6;
constexpr int kWoMaxM = 64;       // the X' atoms of more rows would leave room for fewer than 3 stages
constexpr int kWoThreads = 320;   // producer, MMA issuer, 4 epilogue warps, 4 dequant warps
constexpr int kWoTableBytes = 256 * 32 * 4;

// A stage: W' codes (16 KB), their scale factors (1 KB), X' (mp rows x 256 bf16 as four atoms).
__host__ __device__ constexpr int wo_stage_bytes(int mp) { return 128 * kBKBytes + 1024 + mp * 512; }

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Value of an E2M1 code (bit 3 sign; magnitude index m: 0, 0.5, then (1 + (m & 1) / 2) * 2^(m / 2 - 1)).
__device__ __forceinline__ float e2m1_to_float(uint32_t code) {
    const uint32_t m = code & 7u;
    const float v = m == 0 ? 0.0f
                  : m == 1 ? 0.5f
                           : __uint_as_float(((126u + (m >> 1)) << 23) | ((m & 1u) << 22));
    return (code & 8u) ? -v : v;
}

// bf16 bits of 2^(E - 127): biased exponent E for E >= 1, the subnormal 2^-127 for E = 0.
__device__ __forceinline__ uint32_t bf16_pow2_bits(uint32_t E) { return E ? (E << 7) : 0x0040u; }

__global__ void __launch_bounds__(kWoThreads, 1)
gemm_w4a16_skinny_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                         const __grid_constant__ CUtensorMap ymap, SkinnyArgs g, const uint8_t *__restrict__ wsf) {
    extern __shared__ uint8_t dsmem[];
    __shared__ uint64_t full_bar[kWoMaxStages];
    __shared__ uint64_t empty_bar[kWoMaxStages];
    __shared__ uint64_t a_full[2];     // dequant warps -> MMA: the A buffer holds the K-block
    __shared__ uint64_t a_empty[2];    // MMA -> dequant warps: the MMAs that read the A buffer finished
    __shared__ uint64_t accum_full[2];
    __shared__ uint64_t accum_empty[2];
    __shared__ uint64_t mma_done;
    __shared__ uint32_t tmem_slot;
    __shared__ int32_t s_last;
    __shared__ volatile int failed;

    const int S = g.stages;
    const int mp = g.mp;
    const int stage_bytes = wo_stage_bytes(mp);
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint32_t *table = reinterpret_cast<uint32_t *>(smem + S * stage_bytes);   // [256 code bytes][32 copies]
    uint8_t *sY = smem + S * stage_bytes + kWoTableBytes;
    auto sW = [&](int s) { return smem + s * stage_bytes; };
    auto sSf = [&](int s) { return smem + s * stage_bytes + 128 * kBKBytes; };
    auto sX = [&](int s, int atom) { return smem + s * stage_bytes + 128 * kBKBytes + 1024 + atom * mp * 128; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = g.K;
    const int kq = K / 128;
    const uint32_t num_kb = static_cast<uint32_t>(K / 256);
    const uint32_t C = gridDim.x;
    const uint32_t chunks = g.units / g.gran;
    const uint32_t u_begin = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x) * chunks) / C) * g.gran;
    const uint32_t u_end = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x + 1) * chunks) / C) * g.gran;
    const uint64_t limit = g.wait_limit_ns;

    auto load_w = [&](uint32_t u, int s) {
        const uint32_t tile = u / num_kb;
        const int kb = static_cast<int>(u - tile * num_kb);
        mbar_arrive_expect_tx(&full_bar[s], static_cast<uint32_t>(stage_bytes));
        tma_load_2d(sW(s), &wmap, &full_bar[s], kb * kBKBytes, static_cast<int32_t>(tile * 128));
        bulk_load(sSf(s), wsf + (static_cast<uint64_t>(tile) * kq + 2 * kb) * 512, 1024, &full_bar[s]);
    };
    auto load_x = [&](uint32_t u, int s) {
        const int kb = static_cast<int>(u % num_kb);
#pragma unroll
        for (int a = 0; a < 4; ++a) tma_load_2d(sX(s, a), &xmap, &full_bar[s], kb * 256 + 64 * a, 0);
    };
    const uint32_t pre = min(static_cast<uint32_t>(S), u_end > u_begin ? u_end - u_begin : 0u);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a_full[b], 4);
            mbar_init(&a_empty[b], 1);
            mbar_init(&accum_full[b], 1);
            mbar_init(&accum_empty[b], 4);
        }
        mbar_init(&mma_done, 1);
        failed = 0;
        fence_mbar_init();
        prefetch_tensor_map(&wmap);
        for (uint32_t i = 0; i < pre; ++i) load_w(u_begin + i, static_cast<int>(i));   // the weights: before TMEM
        prefetch_tensor_map(&xmap);
        prefetch_tensor_map(&ymap);
    }
    // the dequant table: entry b holds the two E2M1 values of code byte b (low nibble in the low half)
    // as bf16x2, one copy per bank
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
        const uint32_t byte = static_cast<uint32_t>(i >> 5);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(e2m1_to_float(byte & 15u), e2m1_to_float(byte >> 4));
        table[i] = *reinterpret_cast<uint32_t *>(&b2);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch_dependents();
    const uint32_t tmem = tmem_slot;   // A buffers at columns 0 and 128, accumulators at 256 and 384

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer
            griddep_wait();   // X' (and Y) may belong to the previous kernel in the stream
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
            const uint32_t idesc = idesc_bf16(static_cast<uint32_t>(mp));
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
                    const int ab = j & 1;
                    if (!mbar_wait_or_abort(&full_bar[s], (j / S) & 1, limit, &failed) ||
                        !mbar_wait_or_abort(&a_full[ab], (j >> 1) & 1, limit, &failed)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int q = 0; q < 16; ++q) {   // K = 16 per MMA: atom q / 4, 32 bytes further per step
                        const uint64_t bdesc = sdesc_sw128(smem_u32(sX(s, q >> 2))) + 2 * (q & 3);
                        tc_mma_bf16_ta(tmem + 256 + 128 * b, tmem + 128 * ab + 8 * q, bdesc, idesc,
                                       (first && q == 0) ? 0u : 1u);
                    }
                    tc_commit(&empty_bar[s]);
                    tc_commit(&a_empty[ab]);
                }
                tc_commit(&accum_full[b]);
            }
            tc_commit(&mma_done);
            mbar_wait(&mma_done, 0, kDrainLimitNs);
        }
    } else if (warp >= 6) {
        // ---------------------------------------------------------------- dequant warps (6-9)
        // warp w: TMEM lane quarter w % 4, i.e. weight rows 32 (w % 4) + lane; each K-block in two
        // halves of 128 elements (64 code bytes, four MX groups, 64 TMEM columns)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t *tab = table + lane;
        uint32_t j = 0;
        for (uint32_t u = u_begin; u < u_end; ++u, ++j) {
            const int s = j % S;
            const int ab = j & 1;
            bool ok = mbar_wait_or_abort(&full_bar[s], (j / S) & 1, limit, &failed);
            if (ok && j >= 2) ok = mbar_wait_or_abort(&a_empty[ab], ((j >> 1) - 1) & 1, limit, &failed);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint8_t *row = sW(s) + r * 128;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                uint4 codes[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)   // 16-byte chunk 4h + i of the row, 128-byte swizzle
                    codes[i] = *reinterpret_cast<const uint4 *>(row + (((4 * h + i) ^ (r & 7)) << 4));
                const uint32_t sf4 = *reinterpret_cast<const uint32_t *>(sSf(s) + 512 * h + (r & 31) * 16 + (r >> 5) * 4);
                uint32_t out[64];
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {   // MX group gq: code bytes 16 gq .. 16 gq + 15
                    const uint32_t sb = bf16_pow2_bits((sf4 >> (8 * gq)) & 0xFFu);
                    const uint32_t scale2 = sb | (sb << 16);
                    const uint32_t words[4] = {codes[gq].x, codes[gq].y, codes[gq].z, codes[gq].w};
#pragma unroll
                    for (int wd = 0; wd < 4; ++wd)
#pragma unroll
                        for (int by = 0; by < 4; ++by) {
                            const uint32_t byte = (words[wd] >> (8 * by)) & 0xFFu;
                            out[16 * gq + 4 * wd + by] = bf16x2_mul(tab[byte * 32], scale2);
                        }
                }
                tmem_st64(tmem + (static_cast<uint32_t>(q * 32) << 16) + 128 * ab + 64 * h, out);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[ab]);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-5)
        skinny_epilogue(g, &ymap, tmem + 256, warp, lane, sY, mp, accum_full, accum_empty, &failed, &s_last, limit,
                        u_begin, u_end, num_kb, chunks);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace macaq
