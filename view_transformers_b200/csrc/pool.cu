// Block average pooling P_b of Q and K ("Block-Sparse Global Attention for Efficient
// Multi-View Geometry Transformers", 关键设计 1): the mean of each run of b consecutive
// patch tokens of the concatenated patch sequence, per head, accumulated in fp32.
//
// HBM-bound: every patch row of Q and K is read once (Np * H * d elements each), the
// pooled fp32 tensors are written once: pq as [H, B, d], pk dimension-major as [H, d, B]
// (the layout the score pass of the mask kernel reads with coalesced loads).
// One CTA per (block, Q|K, 32 16-byte chunks of the row = 4 heads in bf16): thousands of
// small CTAs keep the HBM queue full to the end. A warp reads 32 consecutive chunks of a
// row (one coalesced 512-byte transaction); 8 row groups x 4 independent loads per thread
// keep the loads in flight.
#include "common.cuh"

namespace bsa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kChunksPerCta = 32;   // 16-byte chunks of a row per CTA (4 heads in bf16)

// Tensor t = blockIdx.y + y0: t = 0 pools q into pq ([H][B][d]); t = 1 pools k into pk,
// dimension-major ([H][d][B]).
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(Geo g, const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ pq,
            float* __restrict__ pk, int y0) {
    extern __shared__ float red[];  // [ngroups][per_round * V] partial sums
    constexpr int V = Vec16<T>::n;
    const int j = blockIdx.x;
    const int t = blockIdx.y + y0;
    const T* src = t == 0 ? q : k;
    float* dst = t == 0 ? pq : pk;
    const bool dim_major = t == 1;
    const int row_elems = g.H * g.d;
    const int chunks = row_elems / V;                     // 16-byte chunks per row
    const int cbeg = blockIdx.z * kChunksPerCta;          // this CTA's chunks of every row
    const int cend = min(chunks, cbeg + kChunksPerCta);
    const int per_round = min(cend - cbeg, kPoolThreads); // chunks covered per round
    const int ngroups = kPoolThreads / per_round;         // row groups per round
    const int lo = j * g.b;
    const int hi = min(lo + g.b, g.Np);
    const float count = (float)(hi - lo);
    const int gi = threadIdx.x / per_round;
    const int ci = threadIdx.x % per_round;

    for (int c0 = cbeg; c0 < cend; c0 += per_round) {
        const int c = c0 + ci;
        if (gi < ngroups && c < cend) {
            float acc[V];
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = 0.f;
            int p = lo + gi;
            for (; p + 3 * ngroups < hi; p += 4 * ngroups) {   // four independent loads in flight
                float x[4][V];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    Vec16<T>::load(src + (size_t)patch_row(g, p + u * ngroups) * row_elems + c * V, x[u]);
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] += x[u][e];
            }
            for (; p < hi; p += ngroups) {
                float x[V];
                Vec16<T>::load(src + (size_t)patch_row(g, p) * row_elems + c * V, x);
#pragma unroll
                for (int e = 0; e < V; ++e) acc[e] += x[e];
            }
            float* r = red + (size_t)gi * per_round * V + ci * V;
#pragma unroll
            for (int e = 0; e < V; ++e) r[e] = acc[e];
        }
        __syncthreads();
        const int width = min(per_round, cend - c0) * V;
        for (int e = threadIdx.x; e < width; e += kPoolThreads) {
            float s = 0.f;
            for (int gg = 0; gg < ngroups; ++gg) s += red[(size_t)gg * per_round * V + e];
            const int el = c0 * V + e;
            const int h = el / g.d;
            const int dd = el - h * g.d;
            const size_t at = !dim_major ? ((size_t)h * g.B + j) * g.d + dd     // [H][B][d]
                                         : ((size_t)h * g.d + dd) * g.B + j;    // [H][d][B]
            dst[at] = s / count;
        }
        __syncthreads();
    }
}

}  // namespace

namespace {
// Tensors y0 .. y0 + tensors - 1 (0: q -> pq, 1: k -> pk dimension-major).
cudaError_t launch_pool_tensors(const Geo& g, bsa_dtype dt, int y0, int tensors, const void* q, const void* k,
                                float* pq, float* pk, cudaStream_t st) {
    const int V = dt == BSA_BF16 ? 8 : 4;
    const int chunks = g.H * g.d / V;
    const size_t smem = (size_t)kPoolThreads * V * sizeof(float);   // ngroups x per_round <= 256 chunks
    const dim3 grid(g.B, tensors, (chunks + kChunksPerCta - 1) / kChunksPerCta);
    if (dt == BSA_BF16) {
        pool_kernel<__nv_bfloat16><<<grid, kPoolThreads, smem, st>>>(
            g, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), pq, pk, y0);
    } else {
        pool_kernel<float><<<grid, kPoolThreads, smem, st>>>(
            g, static_cast<const float*>(q), static_cast<const float*>(k), pq, pk, y0);
    }
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_pool(const Geo& g, bsa_dtype dt, const void* q, const void* k, float* pq,
                        float* pk, cudaStream_t st) {
    return launch_pool_tensors(g, dt, 0, 2, q, k, pq, pk, st);
}

// P_b(V), dimension-major [H][d][B] (the layout the drift-score kernel stages in shared memory):
// the K branch of the same kernel, run on V alone.
cudaError_t launch_pool_v(const Geo& g, bsa_dtype dt, const void* v, float* pv, cudaStream_t st) {
    return launch_pool_tensors(g, dt, 1, 1, nullptr, v, nullptr, pv, st);
}

}  // namespace bsa
