// swiglu.cuh -- the down projection's activation quantization fused after the gate/up GEMM.
//
// In a SwiGLU MLP the down projection's input is H = silu(G) * U, with G and U the gate and up
// projections of the same X. MACaQ transforms and quantizes the input of every linear (page
// "Huawei's research lab in Switzerland open-sources the four-bit quantization tool MACaQ ..."
// (aipolix.com), paragraph 2), so H goes through the down projection's per-channel 1/s, block
// Hadamard and MXFP4 before its GEMM. Here that happens on the gate/up GEMM's fp32 accumulators:
//     h   = fl32( fl32( g / fl32(1 + exp32(-g)) ) * u )
//     H'  = MXFP4( h * diag(1/s_down) * H_b )          (the act_quant arithmetic, unchanged)
// exp32 is one fixed fp32 evaluation of exp, so that the codes are a defined function of (g, u):
// Cody and Waite's reduction (W. J. Cody, W. Waite, "Software Manual for the Elementary Functions",
// 1980) n = rint(x log2 e), r = (x - n C1) - n C2 with ln 2 = C1 + C2 (C1 short, so n C1 is exact),
// the Taylor polynomial sum_{k<=6} r^k / k! by Horner's rule, then p * 2^n; x is clamped to
// [-100, 88] so 2^n is a representable float. Every step is one fp32 operation rounded to nearest;
// no multiply-add is contracted.
//
// Column layout of the gate/up GEMM (N = 2I outputs): weight rows are interleaved in blocks of 64,
// gate rows [64j, 64j + 64) then up rows [64j, 64j + 64), so output columns [128j, 128j + 64) are
// G[:, 64j..] and [128j + 64, 128j + 128) are U[:, 64j..]. A thread holding 64 consecutive
// intermediate channels of one row (one gate block and its up block) produces two whole MX groups.
#pragma once

#include "groups.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace macaq {

__device__ __forceinline__ float exp32_cw(float x) {
    const float log2e = __uint_as_float(0x3FB8AA3Bu);   // 1.44269504
    const float c1 = __uint_as_float(0x3F317200u);      // 0.693145751953125 (ln 2, high part)
    const float c2 = __uint_as_float(0x35BFBE8Eu);      // 1.42860677e-06 (ln 2 - c1)
    const float inv_fact[7] = {1.0f, 1.0f, 0.5f, __uint_as_float(0x3E2AAAABu), __uint_as_float(0x3D2AAAABu),
                               __uint_as_float(0x3C088889u), __uint_as_float(0x3AB60B61u)};  // 1/k!, k = 0..6
    x = x < -100.0f ? -100.0f : x;
    x = x > 88.0f ? 88.0f : x;
    const float nf = rintf(__fmul_rn(x, log2e));
    float r = __fsub_rn(x, __fmul_rn(nf, c1));
    r = __fsub_rn(r, __fmul_rn(nf, c2));
    float p = inv_fact[6];
#pragma unroll
    for (int k = 5; k >= 0; --k) p = __fadd_rn(__fmul_rn(p, r), inv_fact[k]);
    const int n = static_cast<int>(nf);                                      // in [-145, 127]
    const float scale = n >= -126 ? __uint_as_float(static_cast<uint32_t>(n + 127) << 23)
                                  : __uint_as_float(1u << (n + 149));        // 2^n, subnormal below -126
    return __fmul_rn(p, scale);
}

__device__ __forceinline__ float swiglu32(float g, float u) {
    const float e = exp32_cw(-g);
    const float s = __fdiv_rn(g, __fadd_rn(1.0f, e));
    return __fmul_rn(s, u);
}

// 64 consecutive intermediate channels of one row: gate g[0..63] and up u[0..63] (fp32, as raw bits
// from TMEM or memory), the down projection's multipliers inv_s[0..63] (nullptr: 1) -> two MX groups
// (32 code bytes, two E8M0 exponents). The Hadamard block b <= 64 stays inside the thread: stages
// h = 1 .. 16 on each group, then h = 32 across the two groups (b = 64).
template <int kB>
__device__ __forceinline__ void swiglu_quant64(const uint32_t (&g)[64], const uint32_t (&u)[64], const float *inv_s,
                                               uint4 (&codes)[2], uint32_t (&E8)[2]) {
    static_assert(kB == 1 || kB == 16 || kB == 32 || kB == 64, "Hadamard block of the fused epilogue");
    uint64_t p[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int k = 32 * h + 2 * i;
            p[h][i] = pk2(swiglu32(__uint_as_float(g[k]), __uint_as_float(u[k])),
                          swiglu32(__uint_as_float(g[k + 1]), __uint_as_float(u[k + 1])));
        }
    if (inv_s != nullptr) {
        const float4 *mp = reinterpret_cast<const float4 *>(inv_s);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 f = __ldg(mp + 8 * h + i);
                p[h][2 * i] = mul2(p[h][2 * i], pk2(f.x, f.y));
                p[h][2 * i + 1] = mul2(p[h][2 * i + 1], pk2(f.z, f.w));
            }
    }
    if constexpr (kB > 1) {
        fwht_in_thread<kB < 32 ? kB : 32>(p[0]);
        fwht_in_thread<kB < 32 ? kB : 32>(p[1]);
        if constexpr (kB == 64) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint64_t a = p[0][i], c = p[1][i];
                p[0][i] = add2(a, c);
                p[1][i] = sub2(a, c);
            }
        }
    }
    mx_encode_group(p[0], codes[0], E8[0]);
    mx_encode_group(p[1], codes[1], E8[1]);
}

// Destination of the quantized down-projection input.
struct SwigluOut {
    const float *inv_s;   // [I] down projection multipliers 1/s, or nullptr
    uint8_t *hq;          // [M, I/2] codes
    uint8_t *hsf;         // tiled SF of M rows (padding rows written as 0)
    int32_t I;            // intermediate channels (N / 2)
    int32_t rows_sf;      // rows of the SF buffer: ceil(M / 128) * 128
};

// Stores the block of intermediate channels [c0, c0 + 64) of row m: 32 code bytes (rows < M) and the
// two E8M0 bytes (rows < rows_sf; padding rows get 0).
__device__ __forceinline__ void store_swiglu64(const SwigluOut &o, int64_t m, int64_t M, int32_t c0, const uint4 (&codes)[2],
                                               const uint32_t (&E8)[2]) {
    if (m < M) {
        uint4 *dst = reinterpret_cast<uint4 *>(o.hq + m * (o.I / 2) + c0 / 2);
        dst[0] = codes[0];
        dst[1] = codes[1];
    }
    if (m < o.rows_sf) {
        const uint16_t v = m < M ? static_cast<uint16_t>(E8[0] | (E8[1] << 8)) : 0;
        *reinterpret_cast<uint16_t *>(o.hsf + sf_offset(static_cast<uint32_t>(m), static_cast<uint32_t>(c0 / 32),
                                                         static_cast<uint32_t>(o.I / 128))) = v;
    }
}

// The same computation as a kernel of its own, on a gate/up output already in memory (fp32 [M, 2I],
// blocks of 64 interleaved as above): one thread per (row, 64-channel block), grid-stride. Used for
// the shapes whose GEMM does not run the fused epilogue.
template <int kB>
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const float *gu, int64_t M, SwigluOut o) {
    griddep_wait();
    griddep_launch_dependents();
    const int64_t blocks = o.I / 64;
    const int64_t rows = o.rows_sf;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < rows * blocks;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / blocks;
        const int32_t j = static_cast<int32_t>(i - m * blocks);
        uint32_t g[64], u[64];
        if (m < M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(gu + m * (2 * static_cast<int64_t>(o.I)) + 128 * j);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint4 a = src[k], b = src[16 + k];
                g[4 * k] = a.x, g[4 * k + 1] = a.y, g[4 * k + 2] = a.z, g[4 * k + 3] = a.w;
                u[4 * k] = b.x, u[4 * k + 1] = b.y, u[4 * k + 2] = b.z, u[4 * k + 3] = b.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 64; ++k) g[k] = u[k] = 0u;
        }
        uint4 codes[2];
        uint32_t E8[2];
        swiglu_quant64<kB>(g, u, o.inv_s == nullptr ? nullptr : o.inv_s + 64 * j, codes, E8);
        store_swiglu64(o, m, M, 64 * j, codes, E8);
    }
}

}  // namespace macaq
