// flip.cuh -- Flip-Refinement of prepared MXFP4 weights (offline).
//
// Page "Huawei's research lab in Switzerland open-sources the four-bit quantization tool MACaQ for
// running models locally" (aipolix.com), paragraph 3: a coordinate-descent step, guided by the
// Hessian, that moves single FP4 codes to the neighbouring representable values. Per weight row:
//   w      the row's transformed fp32 weights, exactly as weight preparation computes them;
//   w_hat  the codes' values at the row's E8M0 scales (the scales never change);
//   L      = (w_hat - w)^T H (w_hat - w) with H symmetric (X'^T X' of the layer's transformed inputs).
// g = H (w_hat - w) is kept in float64. For k = 0 .. K-1 (sweeps times) the two neighbouring signed
// grid values are tried, the lower first; a move by d changes L by d (2 g[k] + d H[k][k]); the better
// one (the upper only if strictly better) is taken when that is negative, and g += d H[k][:]. Each
// step is one float64 operation in the order written, so the result is one defined set of codes.
//
// B200 mapping: a CTA refines R rows at once (the rows share every read of H). Shared memory holds,
// per row, g (float64), w (fp32), the 4-bit codes (one per byte) and the exponents. Phase 1 forms g
// with k outermost: every thread keeps the float64 sums of its columns for all R rows in registers
// and reads row k of H (coalesced; by symmetry it is column k), so each g[i] is summed over k in
// order. Phase 2 walks k: R threads take the decisions, and when a move is taken every thread adds
// d * H[k][i] to its columns' g. H (fp32, K x K) is read from L2 and HBM by all CTAs.
#pragma once

#include <cuda_bf16.h>

#include "groups.cuh"
#include "ptx.cuh"

namespace macaq {

struct FlipArgs {
    const uint16_t *w;    // bf16 [N, K]
    const float *s;       // [K] per-channel scale, or nullptr
    const float *h;       // fp32 [K, K], symmetric
    uint8_t *wq;          // [N, K/2] codes, refined in place
    const uint8_t *wsf;   // tiled SF of N rows (read)
    int32_t *flips;       // [N] accepted moves per row, or nullptr
    int32_t N, K, sweeps, had_block;
};

constexpr int kFlipThreads = 256;

__host__ __device__ constexpr size_t flip_smem_bytes(int R, int K) {
    return static_cast<size_t>(R) * K * (8 + 4 + 1) + static_cast<size_t>(R) * (K / 32) + 64;
}

__device__ __forceinline__ double pow2_f64(int e) { return __longlong_as_double(static_cast<long long>(e + 1023) << 52); }

// E2M1 value of a code, exact in float64: magnitude index m = 0, 1 are 0 and 0.5; m >= 2 is
// (1 + (m & 1) / 2) * 2^(m / 2 - 1); bit 3 is the sign (so code 0x8 is -0).
__device__ __forceinline__ double e2m1_value_f64(uint32_t code) {
    const uint32_t m = code & 7u;
    const double v = m < 2 ? 0.5 * static_cast<double>(m)
                           : (1.0 + 0.5 * static_cast<double>(m & 1u)) * pow2_f64(static_cast<int>(m >> 1) - 1);
    return (code & 8u) ? -v : v;
}

__device__ __forceinline__ int e2m1_t(uint32_t code) { return (code & 8u) ? -static_cast<int>(code & 7u) : static_cast<int>(code & 7u); }
__device__ __forceinline__ uint32_t e2m1_from_t(int t) { return t > 0 ? static_cast<uint32_t>(t) : (t < 0 ? static_cast<uint32_t>(8 - t) : 0u); }

template <int kCols, int kR>
__global__ void __launch_bounds__(kFlipThreads, 1) flip_refine_kernel(FlipArgs a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    const int K = a.K;
    double *sg = reinterpret_cast<double *>(dsm);                   // [kR][K]
    float *sw = reinterpret_cast<float *>(sg + kR * K);             // [kR][K]
    uint8_t *sc = reinterpret_cast<uint8_t *>(sw + kR * K);         // [kR][K] codes
    int8_t *sE = reinterpret_cast<int8_t *>(sc + kR * K);           // [kR][K/32] scale exponent - 127
    // the decisions of step k live in s_d[k & 1]: a thread writes the slot of step k + 2 only after
    // every thread has passed the decision barrier of step k + 1, so the slot of step k is no longer read
    __shared__ double s_d[2][kR];
    __shared__ int32_t s_n[kR];
    const int tid = threadIdx.x;
    const int kg = K / 32, kq = K / 128;
    griddep_wait();
    griddep_launch_dependents();

    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kR; base < a.N; base += static_cast<int64_t>(gridDim.x) * kR) {
        const int rows = static_cast<int>(min(static_cast<int64_t>(kR), a.N - base));
        // ---------------------------------------------------------------- phase 0: inputs
        for (int idx = tid; idx < kR * K; idx += kFlipThreads) {
            const int r = idx / K, k = idx - r * K;
            if (r < rows) {
                const int64_t n = base + r;
                sc[idx] = static_cast<uint8_t>((a.wq[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 15u);
                float x = __uint_as_float(static_cast<uint32_t>(a.w[n * K + k]) << 16);
                if (a.s != nullptr) x = __fmul_rn(x, a.s[k]);
                sw[idx] = x;
            } else {
                sc[idx] = 0;
                sw[idx] = 0.0f;
            }
        }
        for (int idx = tid; idx < kR * kg; idx += kFlipThreads) {
            const int r = idx / kg, c = idx - r * kg;
            sE[idx] = r < rows ? static_cast<int8_t>(static_cast<int>(a.wsf[sf_offset(static_cast<uint32_t>(base + r), c, kq)]) - 127)
                               : static_cast<int8_t>(0);
        }
        if (tid < kR) s_n[tid] = 0;
        __syncthreads();
        // the weight transform of preparation: butterfly stages h = 1, 2, ..., b/2, then the exact 1/b
        for (int hs = 1; hs < a.had_block; hs <<= 1) {
            for (int p = tid; p < kR * (K / 2); p += kFlipThreads) {
                const int r = p / (K / 2), q = p - r * (K / 2);
                const int j = (q / hs) * 2 * hs + (q % hs);
                const float x = sw[r * K + j], y = sw[r * K + j + hs];
                sw[r * K + j] = __fadd_rn(x, y);
                sw[r * K + j + hs] = __fsub_rn(x, y);
            }
            __syncthreads();
        }
        if (a.had_block > 1) {
            const float inv_b = 1.0f / static_cast<float>(a.had_block);   // a power of two: exact
            for (int idx = tid; idx < kR * K; idx += kFlipThreads) sw[idx] = __fmul_rn(sw[idx], inv_b);
            __syncthreads();
        }

        // ---------------------------------------------------------------- phase 1: g = H (w_hat - w)
        double acc[kCols][kR];
#pragma unroll
        for (int j = 0; j < kCols; ++j)
#pragma unroll
            for (int r = 0; r < kR; ++r) acc[j][r] = 0.0;
        for (int k = 0; k < K; ++k) {
            double e[kR];
#pragma unroll
            for (int r = 0; r < kR; ++r)
                e[r] = __dsub_rn(__dmul_rn(e2m1_value_f64(sc[r * K + k]), pow2_f64(sE[r * kg + k / 32])),
                                 static_cast<double>(sw[r * K + k]));
            const float *hrow = a.h + static_cast<int64_t>(k) * K;
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                const int i = tid + j * kFlipThreads;
                if (i < K) {
                    const double hv = static_cast<double>(__ldg(hrow + i));
#pragma unroll
                    for (int r = 0; r < kR; ++r) acc[j][r] = __dadd_rn(acc[j][r], __dmul_rn(hv, e[r]));
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kCols; ++j) {
            const int i = tid + j * kFlipThreads;
            if (i < K)
#pragma unroll
                for (int r = 0; r < kR; ++r) sg[r * K + i] = acc[j][r];
        }
        __syncthreads();

        // ---------------------------------------------------------------- phase 2: the sweeps
        for (int sw_i = 0; sw_i < a.sweeps; ++sw_i) {
            for (int k = 0; k < K; ++k) {
                if (tid < kR) {
                    const int r = tid;
                    double best_d = 0.0;
                    if (r < rows) {
                        const uint32_t c = sc[r * K + k];
                        const int t = e2m1_t(c);
                        const double scale = pow2_f64(sE[r * kg + k / 32]);
                        const double v = __dmul_rn(e2m1_value_f64(c), scale);
                        const double hkk = static_cast<double>(__ldg(a.h + static_cast<int64_t>(k) * K + k));
                        const double two_g = __dmul_rn(2.0, sg[r * K + k]);
                        int best_t = t;
                        double best_dl = 0.0;
#pragma unroll
                        for (int dir = -1; dir <= 1; dir += 2) {
                            const int tc = t + dir;
                            if (tc < -7 || tc > 7) continue;
                            const double d = __dsub_rn(__dmul_rn(e2m1_value_f64(e2m1_from_t(tc)), scale), v);
                            const double dl = __dmul_rn(d, __dadd_rn(two_g, __dmul_rn(d, hkk)));
                            if (dl < best_dl) {
                                best_dl = dl;
                                best_d = d;
                                best_t = tc;
                            }
                        }
                        if (best_t != t) {
                            sc[r * K + k] = static_cast<uint8_t>(e2m1_from_t(best_t));
                            ++s_n[r];
                        } else {
                            best_d = 0.0;
                        }
                    }
                    s_d[k & 1][r] = best_d;
                }
                __syncthreads();
                bool any = false;
#pragma unroll
                for (int r = 0; r < kR; ++r) any |= s_d[k & 1][r] != 0.0;
                if (any) {   // uniform: every thread read the same s_d
                    const float *hrow = a.h + static_cast<int64_t>(k) * K;
                    double d[kR];
#pragma unroll
                    for (int r = 0; r < kR; ++r) d[r] = s_d[k & 1][r];
#pragma unroll
                    for (int j = 0; j < kCols; ++j) {
                        const int i = tid + j * kFlipThreads;
                        if (i < K) {
                            const double hv = static_cast<double>(__ldg(hrow + i));
#pragma unroll
                            for (int r = 0; r < kR; ++r)
                                if (d[r] != 0.0) sg[r * K + i] = __dadd_rn(sg[r * K + i], __dmul_rn(d[r], hv));
                        }
                    }
                    __syncthreads();
                }
            }
        }

        // ---------------------------------------------------------------- phase 3: write back
        for (int idx = tid; idx < rows * (K / 2); idx += kFlipThreads) {
            const int r = idx / (K / 2), j = idx - r * (K / 2);
            a.wq[(base + r) * (K / 2) + j] = static_cast<uint8_t>(sc[r * K + 2 * j] | (sc[r * K + 2 * j + 1] << 4));
        }
        if (a.flips != nullptr && tid < rows) a.flips[base + tid] = s_n[tid];
        __syncthreads();
    }
}

}  // namespace macaq
