// Warp-level "k smallest keys, ties to the lower index" shared by the block selectors: a radix
// select over 8-bit digits (most significant first, a 256-bin shared-memory histogram per
// pass), then the kept indices in ascending order by ballots. Integer work: exact.
#pragma once

#include <cstdint>

namespace bsa {

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// One warp: of keys[0, n) (shared memory; 32- or 64-bit unsigned keys), keep the `need`
// entries with the smallest (key, index). Writes the kept indices in ascending order to out[0, count) and, when
// `bits` is not null, the row's kept-block bits (word w = blocks 32w .. 32w+31). `hist` is
// 256 words of shared memory owned by the warp. Returns the count (min(need, n)).
template <typename Key>
__device__ int warp_select_smallest(const Key* keys, int n, int need, uint16_t* out, uint32_t* bits,
                                    unsigned* hist) {
    const int lane = threadIdx.x & 31;
    Key thr = 0;
    int take_eq = 0;   // entries equal to thr that are kept, lowest indices first
    const bool all = need >= n;
    if (!all && need > 0) {
        Key prefix = 0, pmask = 0;
        int rem = need;
        for (int shift = 8 * (int)sizeof(Key) - 8; shift >= 0; shift -= 8) {
            for (int b = lane; b < 256; b += 32) hist[b] = 0u;
            __syncwarp();
            for (int j = lane; j < n; j += 32) {
                const Key u = keys[j];
                if ((u & pmask) == prefix) atomicAdd(&hist[(unsigned)(u >> shift) & 255u], 1u);
            }
            __syncwarp();
            // lane l owns digits 8l .. 8l+7; the digit where the running count reaches rem
            unsigned c[8], local = 0u;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c[q] = hist[8 * lane + q];
                local += c[q];
            }
            unsigned incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const unsigned excl = incl - local;
            const unsigned hit = __ballot_sync(0xffffffffu, excl < (unsigned)rem && (unsigned)rem <= incl);
            const int src = __ffs(hit) - 1;   // rem <= number of candidates, so one lane hits
            int digit = 0;
            unsigned before = 0u;
            if (lane == src) {
                unsigned acc = excl;
                int q = 0;
                while (q < 7 && acc + c[q] < (unsigned)rem) acc += c[q++];
                digit = 8 * lane + q;
                before = acc;
            }
            digit = __shfl_sync(0xffffffffu, digit, src);
            before = __shfl_sync(0xffffffffu, before, src);
            rem -= (int)before;
            prefix |= (Key)digit << shift;
            pmask |= (Key)0xff << shift;
            __syncwarp();
        }
        thr = prefix;
        take_eq = rem;
    }
    int pos = 0, eq_seen = 0;
    const unsigned lt_mask = lanemask_lt();
    for (int base = 0; base < n; base += 32) {
        const int j = base + lane;
        const bool valid = j < n;
        const Key u = valid ? keys[j] : ~(Key)0;
        bool sel;
        if (all) {
            sel = valid;
        } else {
            const unsigned eqm = __ballot_sync(0xffffffffu, valid && u == thr && need > 0);
            const int r = eq_seen + __popc(eqm & lt_mask);
            sel = need > 0 && valid && (u < thr || (u == thr && r < take_eq));
            eq_seen += __popc(eqm);
        }
        const unsigned sm = __ballot_sync(0xffffffffu, sel);
        if (sel && out != nullptr) out[pos + __popc(sm & lt_mask)] = (uint16_t)j;
        pos += __popc(sm);
        if (bits != nullptr && lane == 0) bits[base >> 5] = sm;
    }
    return pos;
}

}  // namespace bsa
