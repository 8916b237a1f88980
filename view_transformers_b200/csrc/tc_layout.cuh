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
    size_t qp, kp, vp;   // byte offsets of the patch arrays   [H][np_pad][64]
    size_t qs, ks, vs;   // byte offsets of the special arrays [H][ns_pad][64]
    size_t bytes;        // total
};

__host__ __device__ inline PackedLayout packed_layout(const Geo& g) {
    PackedLayout pl;
    pl.np_pad = (g.Np + 127) / 128 * 128;
    pl.ns_pad = (g.Ns + 127) / 128 * 128;
    const size_t patch = (size_t)g.H * pl.np_pad * 128;
    const size_t spec = (size_t)g.H * pl.ns_pad * 128;
    pl.qp = 0;
    pl.kp = pl.qp + patch;
    pl.vp = pl.kp + patch;
    pl.qs = pl.vp + patch;
    pl.ks = pl.qs + spec;
    pl.vs = pl.ks + spec;
    pl.bytes = pl.vs + spec;
    return pl;
}

}  // namespace bsa
