// Byte layout of the packed workspace shared by the packing kernel and the tensor-core
// attention kernels (host and device).
#pragma once

#include <cstddef>
#include <cstdint>

#include "common.cuh"

namespace bsa {

struct PackedLayout {
    int np_pad;          // patch rows per head, multiple of 128
    int ns_pad;          // special rows per head, multiple of 128 (0 without specials)
    int nsplit;          // key-range splits of the special-query attention
    size_t qp, kp, vp;   // byte offsets of the patch arrays   [H][np_pad][64]
    size_t qs, ks, vs;   // byte offsets of the special arrays [H][ns_pad][64]
    size_t spart;        // fp32 [nsplit][H][ns_pad][64] partial outputs of special queries
    size_t slse;         // fp32 [nsplit][H][ns_pad] their log-sum-exp values
    size_t bytes;        // total
};

// Key-range splits of the special-query attention (units = query tiles x heads CTAs per
// split, n_all key tiles): the fewest splits, at most 128 key tiles each, whose CTAs fill
// at least 95% of their last wave on a B200 (148 SMs, 2 attention CTAs resident per SM);
// each split keeps at least 8 key tiles, and the best fill found is taken when none reaches
// 95%.
__host__ __device__ inline int special_splits(int units, int n_all) {
    constexpr int kSlots = 148 * 2;
    const int lo = (n_all + 127) / 128 > 1 ? (n_all + 127) / 128 : 1;
    int hi = n_all / 8 < 64 ? n_all / 8 : 64;
    hi = hi > lo ? hi : lo;
    int best = lo;
    double best_fill = 0.0;
    for (int ns = lo; ns <= hi; ++ns) {
        const long long ctas = (long long)units * ns;
        const long long waves = (ctas + kSlots - 1) / kSlots;
        const double fill = (double)ctas / (double)(waves * kSlots);
        if (fill >= 0.95) return ns;
        if (fill > best_fill) { best = ns; best_fill = fill; }
    }
    return best;
}

__host__ __device__ inline PackedLayout packed_layout(const Geo& g) {
    PackedLayout pl;
    pl.np_pad = (g.Np + 127) / 128 * 128;
    pl.ns_pad = (g.Ns + 127) / 128 * 128;
    // special queries see every key: the key range is split across CTAs
    const int n_all = pl.ns_pad / 128 + pl.np_pad / 128;
    pl.nsplit = g.Ns == 0 ? 0 : special_splits(pl.ns_pad / 128 * g.H, n_all);
    const size_t patch = (size_t)g.H * pl.np_pad * 128;
    const size_t spec = (size_t)g.H * pl.ns_pad * 128;
    pl.qp = 0;
    pl.kp = pl.qp + patch;
    pl.vp = pl.kp + patch;
    pl.qs = pl.vp + patch;
    pl.ks = pl.qs + spec;
    pl.vs = pl.ks + spec;
    pl.spart = pl.vs + spec;
    pl.slse = pl.spart + (size_t)pl.nsplit * g.H * pl.ns_pad * 64 * 4;
    pl.bytes = pl.slse + ((size_t)pl.nsplit * g.H * pl.ns_pad * 4 + 1023) / 1024 * 1024;
    return pl;
}

// Per-frame packing for the frame-wise attention: per head and frame, the frame's T tokens
// (special tokens included) padded with zero rows to a multiple of 128; Q, K bf16, V fp16.
struct FrameLayout {
    int t_pad;           // rows per (head, frame)
    size_t qf, kf, vf;   // byte offsets of [H][F][t_pad][64]
    size_t bytes;
};

__host__ __device__ inline FrameLayout frame_layout(const Geo& g) {
    FrameLayout fl;
    fl.t_pad = (g.T + 127) / 128 * 128;
    const size_t one = (size_t)g.H * g.F * fl.t_pad * 128;
    fl.qf = 0;
    fl.kf = one;
    fl.vf = 2 * one;
    fl.bytes = 3 * one;
    return fl;
}

}  // namespace bsa
