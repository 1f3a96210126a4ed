// groups.cuh -- row partition of a grouped (MoE) call, read from the device-side offsets.
//
// Rows [off[e], off[e+1]) belong to expert e. Each expert's scale factors start on a fresh
// 128-row tile, so expert e owns SF row tiles [tb[e], tb[e+1]) with tb an exclusive prefix sum of
// ceil(M_e / 128). The quantizer (which writes the SF) and the GEMM (which reads it) both derive
// off[] and tb[] with this one routine, so they agree on every tile even for malformed offsets:
// values are clamped into [0, rows] and made non-decreasing, which keeps every access inside
// macaq_grouped_sf_bytes(rows, E, K).
#pragma once

#include <stdint.h>

namespace macaq {

// Fills s_off[0..E] and s_tb[0..E] in shared memory. offsets == nullptr means one group of all
// rows. Must be called by every thread of the block (contains __syncthreads); warp 0 does the
// scans.
__device__ __forceinline__ void load_group_layout(const int32_t *__restrict__ offsets, int32_t E, int64_t rows,
                                                  int32_t *s_off, int32_t *s_tb) {
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    if (offsets == nullptr) {
        if (tid == 0) {
            s_off[0] = 0;
            s_off[1] = static_cast<int32_t>(rows);
            s_tb[0] = 0;
            s_tb[1] = static_cast<int32_t>((rows + 127) / 128);
        }
        __syncthreads();
        return;
    }
    for (int e = tid; e <= E; e += blockDim.x) {
        int64_t v = offsets[e];
        v = v < 0 ? 0 : (v > rows ? rows : v);
        s_off[e] = static_cast<int32_t>(v);
    }
    __syncthreads();
    if (tid < 32) {
        // running maximum (non-decreasing offsets), chunks of 32 with a carry
        int32_t carry = 0;
        for (int base = 0; base <= E; base += 32) {
            const int e = base + lane;
            int32_t x = (e <= E) ? s_off[e] : 0;
            x = x > carry ? x : carry;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, x, d);
                if (lane >= d) x = x > y ? x : y;
            }
            if (e <= E) s_off[e] = x;
            carry = __shfl_sync(0xffffffffu, x, 31);
        }
        __syncwarp();
        // exclusive prefix of ceil(M_e / 128)
        int32_t acc = 0;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            const int32_t cnt = (e < E) ? (s_off[e + 1] - s_off[e] + 127) >> 7 : 0;
            int32_t x = cnt;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, x, d);
                if (lane >= d) x += y;
            }
            if (e < E) s_tb[e] = acc + x - cnt;
            acc += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) s_tb[E] = acc;
    }
    __syncthreads();
}

// Expert owning row m (the last e with s_off[e] <= m < s_off[e+1]), or -1 when no expert does.
__device__ __forceinline__ int find_group(const int32_t *s_off, int32_t E, int64_t m) {
    if (m < s_off[0] || m >= s_off[E]) return -1;
    int lo = 0, hi = E;  // invariant: s_off[lo] <= m < s_off[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_off[mid] <= m) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Byte offset of scale factor (row r, scale column c) in the tcgen05 block-scale tiling:
// 128 x 4 tiles, row-tile-major then K-tile, (r % 32) * 16 + (r / 32 % 4) * 4 + c % 4 inside.
__device__ __forceinline__ uint64_t sf_offset(uint32_t r, uint32_t c, uint32_t kq /* K / 128 */) {
    const uint32_t rt = r >> 7, rr = r & 127;
    return ((static_cast<uint64_t>(rt) * kq + (c >> 2)) << 9) + ((rr & 31) << 4) + ((rr >> 5) << 2) + (c & 3);
}

}  // namespace macaq
