// Tile helpers shared by the streaming kernels over long rows (emit, the
// dense VJP passes and the support backward): a CTA of 256 threads owns a
// 4096-score tile, 16 scores per thread as four striped float4 accesses, so
// that every warp access covers 512 contiguous bytes.
#pragma once

#include "lapsum_common.cuh"
#include "lapsum_kernels.h"

namespace lapsum {
namespace stream_detail {

constexpr int kThreads = 256;
constexpr int kPer = kStreamTile / kThreads;  // 16

// Swizzled slot of value j (0..15) in a lane's 16-float staging row, so that a
// warp's 16-byte stores of the four float4 groups hit distinct banks.
__device__ __forceinline__ int stage_slot16(int lane, int j) {
    return lane * 16 + ((((j >> 2) ^ (lane >> 1)) & 3) << 2) + (j & 3);
}

template <bool VEC>
__device__ __forceinline__ void load_tile(const float* __restrict__ row, int64_t n, int64_t base,
                                          float (&x)[kPer], bool (&ok)[kPer]) {
    if constexpr (VEC) {
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) {
            const int64_t i0 = base + ((int64_t)q * kThreads + threadIdx.x) * 4;
            if (i0 + 4 <= n) {
                const float4 v = __ldcs(reinterpret_cast<const float4*>(row + i0));
                x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
#pragma unroll
                for (int c = 0; c < 4; ++c) ok[4 * q + c] = true;
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    ok[4 * q + c] = i0 + c < n;
                    x[4 * q + c] = ok[4 * q + c] ? row[i0 + c] : 0.f;
                }
            }
        }
    } else {
        // scalar accesses in the same element order as the float4 path
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int64_t i = base + ((int64_t)(q / 4) * kThreads + threadIdx.x) * 4 + q % 4;
            ok[q] = i < n;
            x[q] = ok[q] ? row[i] : 0.f;
        }
    }
}

template <bool VEC>
__device__ __forceinline__ void store_tile(float* __restrict__ row, int64_t n, int64_t base,
                                           const float (&y)[kPer]) {
    if constexpr (VEC) {
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) {
            const int64_t i0 = base + ((int64_t)q * kThreads + threadIdx.x) * 4;
            if (i0 + 4 <= n) {
                __stcs(reinterpret_cast<float4*>(row + i0),
                       make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (i0 + c < n) row[i0 + c] = y[4 * q + c];
            }
        }
    } else {
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int64_t i = base + ((int64_t)(q / 4) * kThreads + threadIdx.x) * 4 + q % 4;
            if (i < n) row[i] = y[q];
        }
    }
}

// True for exactly one CTA per row: the last to finish.  Release/acquire
// through a fence around the ticket; the winner resets the ticket.
__device__ __forceinline__ bool last_block_of_row(uint32_t* ticket, uint32_t nblocks, int* flag) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(ticket, 1u);
        *flag = (prev == nblocks - 1);
        if (*flag) *ticket = 0u;
    }
    __syncthreads();
    if (*flag) __threadfence();
    return *flag != 0;
}

// Online sums of the VJP's ratio R = sum v f / sum f: per thread (mu, S, Sv)
// with mu the smallest |x| seen, S = sum exp(-(|x| - mu)) and
// Sv = sum v exp(-(|x| - mu)); a smaller |x| rescales the sums once.
// Four scores at a time: a new minimum rescales the fp64 sums once, then the
// four weights are summed in fp32 (each at most 1) and added in fp64.
__device__ __forceinline__ void online_add4(float a0, float a1, float a2, float a3, float v0,
                                            float v1, float v2, float v3, float& mu, double& s,
                                            double& sv) {
    const float m4 = fminf(fminf(a0, a1), fminf(a2, a3));
    if (m4 < mu) {
        const double sc = (mu == INFINITY) ? 0.0 : (double)__expf(m4 - mu);
        s *= sc;
        sv *= sc;
        mu = m4;
    }
    const float w0 = __expf(mu - a0), w1 = __expf(mu - a1), w2 = __expf(mu - a2),
                w3 = __expf(mu - a3);
    s += (double)((w0 + w1) + (w2 + w3));
    sv += (double)(fmaf(w0, v0, w1 * v1) + fmaf(w2, v2, w3 * v3));
}
__device__ __forceinline__ void online_add(float ax, float vv, float& mu, double& s, double& sv) {
    online_add4(ax, INFINITY, INFINITY, INFINITY, vv, 0.f, 0.f, 0.f, mu, s, sv);
}

}  // namespace stream_detail
}  // namespace lapsum
