// moe.cuh -- the weighted top-k combine after a mixture-of-experts down projection.
//
//   out[t, n] = sum over j = 0 .. topk-1 of fl32( w[t, j] * Y[pos[t, j], n] )
//
// Y is the grouped GEMM's bf16 output in expert-sorted row order; pos[t, j] is the row that holds
// token t's j-th expert choice and w[t, j] its router weight. The sum runs in fp32 in the order
// j = 0, 1, ..., starting from +0, with every product and every sum rounded on its own (no
// multiply-add contraction), so the result is one defined fp32 value; bf16 output is its
// round-to-nearest-even cast. A pos value outside [0, y_rows) contributes nothing (a dropped choice).
// HBM-bound: each thread owns 8 consecutive columns (one 16-byte load per chosen row) of one token,
// with the loads of up to 8 choices in flight before their products are added in order.
// Source: glonce.com page on MACaQ, paragraph 5 (grouped matmul for mixture-of-experts layers); the
// combine is the step that returns the grouped GEMM's rows to token order.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace macaq {

struct CombineArgs {
    const uint16_t *y;     // bf16 [y_rows, N]
    const int32_t *pos;    // [T, topk]
    const float *w;        // [T, topk]
    void *out;             // [T, N] bf16 or fp32
    int64_t y_rows;
    int64_t T;
    int32_t topk;
    int32_t N;
    int32_t out_f32;
};

constexpr int kCombineThreads = 256;
constexpr int kCombineBatch = 8;   // choices whose rows are loaded before any of them is added

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__global__ void __launch_bounds__(kCombineThreads) moe_combine_kernel(CombineArgs c) {
    griddep_wait();  // Y, the routing and the output may belong to the previous kernel in the stream
    griddep_launch_dependents();
    const int64_t chunks = c.N / 8;
    const int64_t total = c.T * chunks;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / chunks;
        const int64_t n0 = (i - t * chunks) * 8;
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
        for (int j0 = 0; j0 < c.topk; j0 += kCombineBatch) {
            uint4 v[kCombineBatch];
            float w[kCombineBatch];
            bool live[kCombineBatch];
#pragma unroll
            for (int b = 0; b < kCombineBatch; ++b) {
                const int j = j0 + b;
                live[b] = false;
                if (j < c.topk) {
                    const int64_t p = c.pos[t * c.topk + j];
                    if (p >= 0 && p < c.y_rows) {
                        live[b] = true;
                        w[b] = c.w[t * c.topk + j];
                        v[b] = ld_nc_v4(c.y + p * c.N + n0);
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < kCombineBatch; ++b) {
                if (!live[b]) continue;
                const uint32_t words[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float lo = __uint_as_float(words[k] << 16);
                    const float hi = __uint_as_float(words[k] & 0xFFFF0000u);
                    acc[2 * k] = __fadd_rn(acc[2 * k], __fmul_rn(w[b], lo));
                    acc[2 * k + 1] = __fadd_rn(acc[2 * k + 1], __fmul_rn(w[b], hi));
                }
            }
        }
        if (c.out_f32) {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(c.out) + t * c.N + n0);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
            uint32_t pk[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
                pk[k] = *reinterpret_cast<uint32_t *>(&b2);
            }
            *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(c.out) + t * c.N + n0) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
    }
}

}  // namespace macaq
