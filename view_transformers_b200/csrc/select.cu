// Alternative block selectors that emit the same kept-block lists as bsa_predict_mask, for
// the same block-sparse attention:
//   random_mask_kernel   "Block-Sparse Global Attention for Efficient Multi-View Geometry
//                        Transformers", 消融实验 (图 10), rows "Random": k_h blocks per query
//                        block, uniformly at random without replacement;
//   uniform_mask_kernel  "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
//                        Transformers", 四、1. 均匀采样核: key blocks at a fixed stride;
//   probe_mask_kernel    same page, 四、1. Query-Probe Top-K 核 with the acceleration of 四、3.:
//                        key blocks ranked by the mean query's scores q_bar . P_b(K)_j / sqrt(d)
//                        (the column means of Q K^T / sqrt(d)); the top k_h are kept by every
//                        query block.
//
// The random draw is keyed by Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011), written here from that definition: block j of row
// (h, i) gets the 32-bit key = word 0 at counter (j, i, h, 0) and key (seed low, seed high),
// and a row keeps the k_h blocks with the smallest (key, j) -- a uniformly random subset.
//
// Both the random and the probe selector take "the k smallest 32-bit keys, ties to the lower
// index" of a row, which one warp finds by a radix select (four 8-bit digits, most
// significant first, a 256-bin histogram in shared memory per pass) and then emits in
// ascending index order with ballots. Integer work: results are exact.
#include "common.cuh"
#include "select.cuh"

namespace bsa {
namespace {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;

// Word 0 of Philox4x32-10 at counter (c0, c1, c2, c3) under key (k0, k1).
__device__ __forceinline__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += kPhiloxW0;
            k1 += kPhiloxW1;
        }
        const uint32_t lo0 = kPhiloxM0 * c0, hi0 = __umulhi(kPhiloxM0, c0);
        const uint32_t lo1 = kPhiloxM1 * c2, hi1 = __umulhi(kPhiloxM1, c2);
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    return c0;
}

// Order-preserving 32-bit image of a float, reversed so that the largest score gets the
// smallest key; -0 and +0 share one key.
__device__ __forceinline__ uint32_t descending_key(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);
    const uint32_t up = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ~up;
}

struct SelParams {
    int k[BSA_MAX_HEADS];
    uint32_t seed_lo, seed_hi;
    int stride;
};

constexpr int kSelWarps = 4;

__host__ __device__ inline size_t random_warp_smem(int B) { return ((size_t)B * 4 + 1024 + 15) / 16 * 16; }

// One warp per (head, query block) row: keys into shared memory, then the select.
__global__ void __launch_bounds__(32 * kSelWarps)
random_mask_kernel(Geo g, SelParams sp, uint32_t* __restrict__ mask_bits, uint16_t* __restrict__ kv_idx,
                   int32_t* __restrict__ kv_cnt) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kSelWarps + warp;
    if (row >= (long long)g.H * g.B) return;
    const int h = (int)(row / g.B), i = (int)(row - (long long)h * g.B);
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + warp * random_warp_smem(g.B));
    unsigned* hist = reinterpret_cast<unsigned*>(keys + g.B);
    for (int j = lane; j < g.B; j += 32)
        keys[j] = philox_word0((uint32_t)j, (uint32_t)i, (uint32_t)h, 0u, sp.seed_lo, sp.seed_hi);
    __syncwarp();
    const int words = (g.B + 31) / 32;
    const int cnt = warp_select_smallest(keys, g.B, sp.k[h], kv_idx + (size_t)row * g.B,
                                         mask_bits ? mask_bits + (size_t)row * words : nullptr, hist);
    if (lane == 0) kv_cnt[row] = cnt;
}

// One warp per row: blocks j = 0, s, 2s, ...
__global__ void __launch_bounds__(32 * kSelWarps)
uniform_mask_kernel(Geo g, int stride, uint32_t* __restrict__ mask_bits, uint16_t* __restrict__ kv_idx,
                    int32_t* __restrict__ kv_cnt) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kSelWarps + warp;
    if (row >= (long long)g.H * g.B) return;
    const int words = (g.B + 31) / 32;
    const unsigned lt_mask = lanemask_lt();
    int pos = 0;
    for (int base = 0; base < g.B; base += 32) {
        const int j = base + lane;
        const bool sel = j < g.B && j % stride == 0;
        const unsigned sm = __ballot_sync(0xffffffffu, sel);
        if (sel) kv_idx[(size_t)row * g.B + pos + __popc(sm & lt_mask)] = (uint16_t)j;
        pos += __popc(sm);
        if (mask_bits != nullptr && lane == 0) mask_bits[(size_t)row * words + (base >> 5)] = sm;
    }
    if (lane == 0) kv_cnt[row] = pos;
}

constexpr int kProbeThreads = 256;
constexpr int kProbeRows = 64;   // query-block rows written per CTA

// Shared-memory layout of the probe kernel (byte offsets, each 16-byte aligned): keys [B]
// u32, histogram [256] u32, kept list [B] u16, kept bits [ceil(B/32)] u32, fp64 partial sums
// [4][64].
struct ProbeSmem {
    size_t keys, hist, list, bits, part, bytes;
    __host__ __device__ explicit ProbeSmem(int B) {
        auto up16 = [](size_t x) { return (x + 15) / 16 * 16; };
        keys = 0;
        hist = up16((size_t)B * 4);
        list = hist + 1024;
        bits = list + up16((size_t)B * 2);
        part = bits + up16((size_t)(B + 31) / 32 * 4);
        bytes = part + 4 * 64 * 8;
    }
};

// Grid (row chunks, heads). Every CTA of a head computes the mean query, the B probe scores
// and the selection (cheap: B x 64 multiply-adds), then writes its chunk of query-block rows.
__global__ void __launch_bounds__(kProbeThreads)
probe_mask_kernel(Geo g, SelParams sp, const float* __restrict__ pq, const float* __restrict__ pk,
                  uint32_t* __restrict__ mask_bits, uint16_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int h = blockIdx.y;
    const int B = g.B;
    const int words = (B + 31) / 32;
    const ProbeSmem lay(B);
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + lay.keys);
    unsigned* hist = reinterpret_cast<unsigned*>(smem + lay.hist);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + lay.list);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + lay.bits);
    double* part = reinterpret_cast<double*>(smem + lay.part);   // [4][64] partial sums, then q_bar
    __shared__ int count;
    // q_bar = (sum_j |I_j| PQ_j) / Np, in fp64: the mean of the patch queries
    const int d = threadIdx.x & 63, quarter = threadIdx.x >> 6;
    double acc = 0.0;
    const float* pqh = pq + (size_t)h * B * 64;
    for (int j = quarter; j < B; j += 4) {
        const int n = min(g.b, g.Np - j * g.b);
        acc += (double)n * (double)pqh[(size_t)j * 64 + d];
    }
    part[quarter * 64 + d] = acc;
    __syncthreads();
    if (threadIdx.x < 64)
        part[threadIdx.x] = (((part[threadIdx.x] + part[64 + threadIdx.x]) + part[128 + threadIdx.x]) +
                             part[192 + threadIdx.x]) / (double)g.Np;
    __syncthreads();
    // probe score of every key block from the dimension-major pooled K, rounded to fp32
    const float* pkh = pk + (size_t)h * 64 * B;
    for (int j = threadIdx.x; j < B; j += kProbeThreads) {
        double s = 0.0;
#pragma unroll 8
        for (int e = 0; e < 64; ++e) s += part[e] * (double)pkh[(size_t)e * B + j];
        keys[j] = descending_key((float)(s * 0.125));   // 1 / sqrt(64)
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int c = warp_select_smallest(keys, B, sp.k[h], list, bits, hist);
        if (threadIdx.x == 0) count = c;
    }
    __syncthreads();
    const int cnt = count;
    const int i0 = blockIdx.x * kProbeRows, i1 = min(B, i0 + kProbeRows);
    for (int i = i0; i < i1; ++i) {
        const size_t row = (size_t)h * B + i;
        for (int t = threadIdx.x; t < cnt; t += kProbeThreads) kv_idx[row * B + t] = list[t];
        if (mask_bits != nullptr)
            for (int t = threadIdx.x; t < words; t += kProbeThreads) mask_bits[row * words + t] = bits[t];
        if (threadIdx.x == 0) kv_cnt[row] = cnt;
    }
}

SelParams make_params(const Geo& g, const int* k_per_head) {
    SelParams sp{};
    for (int h = 0; h < g.H; ++h) sp.k[h] = k_per_head ? k_per_head[h] : 0;
    return sp;
}

}  // namespace

cudaError_t launch_random_mask(const Geo& g, const int* k_per_head, uint64_t seed, uint32_t* mask_bits,
                               uint16_t* kv_idx, int32_t* kv_cnt, cudaStream_t st) {
    SelParams sp = make_params(g, k_per_head);
    sp.seed_lo = (uint32_t)(seed & 0xffffffffu);
    sp.seed_hi = (uint32_t)(seed >> 32);
    const size_t smem = kSelWarps * random_warp_smem(g.B);
    cudaError_t e = cudaFuncSetAttribute(random_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)g.H * g.B;
    random_mask_kernel<<<(unsigned)((rows + kSelWarps - 1) / kSelWarps), 32 * kSelWarps, smem, st>>>(
        g, sp, mask_bits, kv_idx, kv_cnt);
    return cudaGetLastError();
}

cudaError_t launch_uniform_mask(const Geo& g, int stride, uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                                cudaStream_t st) {
    const long long rows = (long long)g.H * g.B;
    uniform_mask_kernel<<<(unsigned)((rows + kSelWarps - 1) / kSelWarps), 32 * kSelWarps, 0, st>>>(
        g, stride, mask_bits, kv_idx, kv_cnt);
    return cudaGetLastError();
}

cudaError_t launch_probe_mask(const Geo& g, const int* k_per_head, const float* pq, const float* pk,
                              uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt, cudaStream_t st) {
    const SelParams sp = make_params(g, k_per_head);
    const size_t smem = ProbeSmem(g.B).bytes;
    cudaError_t e = cudaFuncSetAttribute(probe_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((g.B + kProbeRows - 1) / kProbeRows, g.H);
    probe_mask_kernel<<<grid, kProbeThreads, smem, st>>>(g, sp, pq, pk, mask_bits, kv_idx, kv_cnt);
    return cudaGetLastError();
}

}  // namespace bsa
