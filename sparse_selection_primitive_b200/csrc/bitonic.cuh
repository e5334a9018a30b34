// Register-resident bitonic sort of u32 keys held in blocked layout: a row of
// NPAD = E * RT keys is spread over RT consecutive threads (RT a multiple of
// 32), E consecutive keys per thread.  Stages whose partner is in the same
// thread compare registers, partners in the same warp exchange by shuffle,
// and partners in other warps go through shared memory (`xch`, E * CTA words).
// Every thread of the CTA must call it (it contains __syncthreads when RT > 32).
#pragma once

#include <cstdint>

namespace lapsum {

template <int E, int RT, int CTA>
__device__ __forceinline__ void bitonic_sort_row(uint32_t (&key)[E], int tid, uint32_t* xch) {
    constexpr int NPAD = E * RT;
#pragma unroll
    for (int size = 2; size <= NPAD; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride < E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ stride;
                    if (pe > e) {
                        const bool asc = (((tid * E + e) & size) == 0);
                        const uint32_t lo = min(key[e], key[pe]), hi = max(key[e], key[pe]);
                        key[e] = asc ? lo : hi;
                        key[pe] = asc ? hi : lo;
                    }
                }
            } else if (stride < 32 * E) {
                const int ls = stride / E;
                const bool asc = (((tid * E) & size) == 0);
                const bool keep_min = (((tid & ls) == 0) == asc);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const uint32_t o = __shfl_xor_sync(0xffffffffu, key[e], ls);
                    key[e] = keep_min ? min(key[e], o) : max(key[e], o);
                }
            } else {
                const int ts = stride / E;
                const bool asc = (((tid * E) & size) == 0);
                const bool keep_min = (((tid & ts) == 0) == asc);
                const int me = threadIdx.x;
                const int partner = me ^ ts;  // rows are aligned to RT, so this stays in the row
#pragma unroll
                for (int e = 0; e < E; ++e) xch[e * CTA + me] = key[e];
                __syncthreads();
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const uint32_t o = xch[e * CTA + partner];
                    key[e] = keep_min ? min(key[e], o) : max(key[e], o);
                }
                __syncthreads();
            }
        }
    }
}

}  // namespace lapsum
