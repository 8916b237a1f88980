// Packing of the bf16 layer inputs into the head-major tile layout read by the tensor-core
// attention kernels (the token split of "Block-Sparse Global Attention for Efficient
// Multi-View Geometry Transformers", 关键设计 3, made physical):
//   patch tokens:   Qp, Kp (bf16), Vp (fp16)  [H][Np_pad][64], row p = patch token p
//   special tokens: Qs, Ks (bf16), Vs (fp16)  [H][Ns_pad][64], row t = special token t
// Np_pad and Ns_pad round up to 128 rows; padding rows are zero. After packing, every
// query tile (128 rows) and key tile (b rows) is one contiguous 2D TMA box, so no tile
// straddles a frame boundary, and V is already in the operand type of the P.V product
// (P is rounded to fp16, whose 11-bit significand keeps the output error well inside
// the bf16 tolerance; bf16 -> fp16 is exact for |v| in [2^-14, 65504]). A V element that
// fp16 cannot hold (|v| >= 65536, inf, NaN) is reported as BSA_ERR_RANGE in the status word.
//
// HBM-bound: Q, K, V read once, written once (plus zero padding).
#include "common.cuh"
#include "tc_layout.cuh"

namespace bsa {
namespace {

// True when a bf16 pair holds an element fp16 cannot hold: magnitude >= 2^16 (bf16 has no
// value between 65280 and 65536, and fp16's largest finite value is 65504), inf or NaN.
__device__ __forceinline__ bool beyond_f16(uint32_t pair) {
    return (pair & 0x7fffu) >= 0x4780u || ((pair >> 16) & 0x7fffu) >= 0x4780u;
}

__device__ __forceinline__ bool beyond_f16(uint4 w) {
    return beyond_f16(w.x) || beyond_f16(w.y) || beyond_f16(w.z) || beyond_f16(w.w);
}

__global__ void __launch_bounds__(256)
pack_kernel(Geo g, PackedLayout pl, const __nv_bfloat16* __restrict__ q,
            const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
            unsigned char* __restrict__ ws, int32_t* status) {
    bool out_of_range = false;
    const int chunks = g.H * 8;                      // 16-byte chunks per token row
    const size_t rows = (size_t)pl.np_pad + pl.ns_pad;
    const size_t total = rows * chunks;
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < total;
         x += (size_t)gridDim.x * blockDim.x) {
        const size_t r = x / chunks;
        const int c = (int)(x - r * chunks);
        const int h = c >> 3;
        const int c8 = c & 7;
        int src_row = -1;
        size_t dst_row;
        size_t base_q, base_k, base_v;
        if (r < (size_t)pl.np_pad) {
            const int p = (int)r;
            if (p < g.Np) src_row = patch_row(g, p);
            dst_row = (size_t)h * pl.np_pad + p;
            base_q = pl.qp; base_k = pl.kp; base_v = pl.vp;
        } else {
            const int t = (int)(r - pl.np_pad);
            if (t < g.Ns) src_row = special_row(g, t);
            dst_row = (size_t)h * pl.ns_pad + t;
            base_q = pl.qs; base_k = pl.ks; base_v = pl.vs;
        }
        uint4 vq = make_uint4(0, 0, 0, 0), vk = vq, vv = vq;
        if (src_row >= 0) {
            const size_t off = (size_t)src_row * g.H * 64 + (size_t)h * 64 + c8 * 8;
            vq = __ldg(reinterpret_cast<const uint4*>(q + off));
            vk = __ldg(reinterpret_cast<const uint4*>(k + off));
            const uint4 w = __ldg(reinterpret_cast<const uint4*>(v + off));
            out_of_range |= beyond_f16(w);
            const uint32_t in[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __half2 hv = __floats2half2_rn(__uint_as_float(in[i] << 16),
                                                     __uint_as_float(in[i] & 0xffff0000u));
                o[i] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            vv = make_uint4(o[0], o[1], o[2], o[3]);
        }
        const size_t dst = dst_row * 128 + c8 * 16;
        *reinterpret_cast<uint4*>(ws + base_q + dst) = vq;
        *reinterpret_cast<uint4*>(ws + base_k + dst) = vk;
        *reinterpret_cast<uint4*>(ws + base_v + dst) = vv;
    }
    if (out_of_range) record_error(status, BSA_ERR_RANGE);
}

// Packing with block pooling folded in: the same copies as pack_kernel, plus the block
// means P_b(Q), P_b(K) of 关键设计 1 taken from the patch rows while they pass through
// registers, so Q and K are read from HBM once for both steps. Written for b dividing 128
// (64 or 128): a 128-row tile then holds 128 / b whole blocks.
//
// Work unit (one CTA each): one 128-row tile (patch tiles first, then special tiles) x one
// pair of heads. 256 threads = 16 chunks of 16 bytes (2 heads x 8) x 16 row phases of 8
// consecutive rows; a row phase therefore never straddles a block. Each thread sums its 8
// rows in fp32 in row order, then the phases of a block are added in phase order, so the
// pooled values do not depend on scheduling. Small units (thousands of CTAs) keep the HBM
// queue full to the end of the pass.
constexpr int kPoolHeads = 2;                 // heads per work unit
constexpr int kPhaseRows = 8;                 // consecutive rows per thread
constexpr int kPhases = 128 / kPhaseRows;     // row phases per tile

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 w) {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 hv = __floats2half2_rn(__uint_as_float(in[i] << 16), __uint_as_float(in[i] & 0xffff0000u));
        o[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void add_bf16x8(float* acc, uint4 w) {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(in[i] << 16);
        acc[2 * i + 1] += __uint_as_float(in[i] & 0xffff0000u);
    }
}

__global__ void __launch_bounds__(256)
pack_pool_kernel(Geo g, PackedLayout pl, const __nv_bfloat16* __restrict__ q,
                 const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                 unsigned char* __restrict__ ws, float* __restrict__ pq, float* __restrict__ pk,
                 int32_t* status) {
    __shared__ float red[2][kPhases][kPoolHeads * 64];   // per-phase sums of Q and K
    bool out_of_range = false;
    const int groups = (g.H + kPoolHeads - 1) / kPoolHeads;
    const int p_tiles = pl.np_pad / 128;
    const int units = (p_tiles + pl.ns_pad / 128) * groups;
    const int c = threadIdx.x % (kPoolHeads * 8);       // chunk within the head group
    const int ph = threadIdx.x / (kPoolHeads * 8);      // row phase
    const int c8 = c & 7;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int tile = u / groups;
        const int h = (u - tile * groups) * kPoolHeads + (c >> 3);
        const bool patch = tile < p_tiles;
        const bool active = h < g.H;
        const int r0 = (patch ? tile : tile - p_tiles) * 128 + ph * kPhaseRows;
        float sq[8], sk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { sq[e] = 0.f; sk[e] = 0.f; }
        if (active) {
            const int limit = patch ? g.Np : g.Ns;
            const size_t dst_base = (size_t)h * (patch ? pl.np_pad : pl.ns_pad);
            unsigned char* oq = ws + (patch ? pl.qp : pl.qs);
            unsigned char* ok = ws + (patch ? pl.kp : pl.ks);
            unsigned char* ov = ws + (patch ? pl.vp : pl.vs);
#pragma unroll 4
            for (int i = 0; i < kPhaseRows; ++i) {
                const int r = r0 + i;
                uint4 vq = make_uint4(0, 0, 0, 0), vk = vq, vv = vq;
                if (r < limit) {
                    const int src_row = patch ? patch_row(g, r) : special_row(g, r);
                    const size_t off = (size_t)src_row * g.H * 64 + (size_t)h * 64 + c8 * 8;
                    vq = __ldg(reinterpret_cast<const uint4*>(q + off));
                    vk = __ldg(reinterpret_cast<const uint4*>(k + off));
                    const uint4 w = __ldg(reinterpret_cast<const uint4*>(v + off));
                    out_of_range |= beyond_f16(w);
                    vv = bf16x8_to_f16x8(w);
                    if (patch) { add_bf16x8(sq, vq); add_bf16x8(sk, vk); }
                }
                const size_t dst = (dst_base + r) * 128 + c8 * 16;
                *reinterpret_cast<uint4*>(oq + dst) = vq;
                *reinterpret_cast<uint4*>(ok + dst) = vk;
                *reinterpret_cast<uint4*>(ov + dst) = vv;
            }
        }
        if (patch) {   // the same for the whole CTA
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                red[0][ph][c * 8 + e] = sq[e];
                red[1][ph][c * 8 + e] = sk[e];
            }
            __syncthreads();
            const int per_tile = 128 / g.b;            // whole blocks in the tile
            const int pb = kPhases / per_tile;         // row phases per block
            const int h0 = (u - tile * groups) * kPoolHeads;
            constexpr int kOut = 2 * kPoolHeads * 64;  // (Q|K) x head x dimension
            for (int x = threadIdx.x; x < per_tile * kOut; x += blockDim.x) {
                const int blk = x / kOut;
                const int t = (x - blk * kOut) / (kPoolHeads * 64);   // 0: Q, 1: K
                const int e = x - blk * kOut - t * kPoolHeads * 64;  // head in group x 64 + dim
                const int j = tile * per_tile + blk;
                const int hh = h0 + e / 64;
                if (j < g.B && hh < g.H) {
                    float sum = 0.f;
                    for (int p2 = blk * pb; p2 < (blk + 1) * pb; ++p2) sum += red[t][p2][e];
                    const int lo = j * g.b;
                    const int hi = min(lo + g.b, g.Np);
                    const float mean = sum / (float)(hi - lo);
                    const int dd = e & 63;
                    if (t == 0) pq[((size_t)hh * g.B + j) * 64 + dd] = mean;   // [H][B][d]
                    else pk[((size_t)hh * 64 + dd) * g.B + j] = mean;          // [H][d][B]
                }
            }
            __syncthreads();
        }
    }
    if (out_of_range) record_error(status, BSA_ERR_RANGE);
}
// Per-frame packing for the frame-wise attention (frame_layout): every token of frame f,
// special tokens included, goes to row r of the (head, frame) slab; rows T .. t_pad-1 are
// zero. Thread order follows the token rows of the input (2 KB of one token per 128 threads
// at 16 heads), so reads are contiguous.
__global__ void __launch_bounds__(256)
pack_frames_kernel(Geo g, FrameLayout fl, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                   unsigned char* __restrict__ ws, int32_t* status) {
    bool out_of_range = false;
    const int chunks = g.H * 8;
    const size_t total = (size_t)g.F * fl.t_pad * chunks;
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < total;
         x += (size_t)gridDim.x * blockDim.x) {
        const size_t fr = x / chunks;                       // (frame, row) pair
        const int c = (int)(x - fr * chunks);
        const int h = c >> 3, c8 = c & 7;
        const int f = (int)(fr / fl.t_pad);
        const int r = (int)(fr - (size_t)f * fl.t_pad);
        uint4 vq = make_uint4(0, 0, 0, 0), vk = vq, vv = vq;
        if (r < g.T) {
            const size_t off = ((size_t)f * g.T + r) * g.H * 64 + (size_t)h * 64 + c8 * 8;
            vq = __ldg(reinterpret_cast<const uint4*>(q + off));
            vk = __ldg(reinterpret_cast<const uint4*>(k + off));
            const uint4 w = __ldg(reinterpret_cast<const uint4*>(v + off));
            out_of_range |= beyond_f16(w);
            vv = bf16x8_to_f16x8(w);
        }
        const size_t dst = (((size_t)h * g.F + f) * fl.t_pad + r) * 128 + c8 * 16;
        *reinterpret_cast<uint4*>(ws + fl.qf + dst) = vq;
        *reinterpret_cast<uint4*>(ws + fl.kf + dst) = vk;
        *reinterpret_cast<uint4*>(ws + fl.vf + dst) = vv;
    }
    if (out_of_range) record_error(status, BSA_ERR_RANGE);
}
}  // namespace

cudaError_t launch_pack_frames(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                               int32_t* status, cudaStream_t st) {
    pack_frames_kernel<<<num_sms() * 8, 256, 0, st>>>(g, frame_layout(g), static_cast<const __nv_bfloat16*>(q),
                                                      static_cast<const __nv_bfloat16*>(k),
                                                      static_cast<const __nv_bfloat16*>(v),
                                                      static_cast<unsigned char*>(ws), status);
    return cudaGetLastError();
}

cudaError_t launch_pack(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                        int32_t* status, cudaStream_t st) {
    const PackedLayout pl = packed_layout(g);
    pack_kernel<<<num_sms() * 8, 256, 0, st>>>(g, pl, static_cast<const __nv_bfloat16*>(q),
                                               static_cast<const __nv_bfloat16*>(k),
                                               static_cast<const __nv_bfloat16*>(v),
                                               static_cast<unsigned char*>(ws), status);
    return cudaGetLastError();
}

cudaError_t launch_pack_pool(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                             float* pq, float* pk, int32_t* status, cudaStream_t st) {
    const PackedLayout pl = packed_layout(g);
    const int groups = (g.H + kPoolHeads - 1) / kPoolHeads;
    const int units = (pl.np_pad / 128 + pl.ns_pad / 128) * groups;
    pack_pool_kernel<<<units, 256, 0, st>>>(
        g, pl, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), static_cast<unsigned char*>(ws), pq, pk, status);
    return cudaGetLastError();
}

}  // namespace bsa
