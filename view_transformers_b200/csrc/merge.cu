// Merge of the two partial attention results of every patch token (flowchart "合并输出"
// of "Block-Sparse Global Attention for Efficient Multi-View Geometry Transformers"):
// one softmax over {special keys} U {kept patch keys}, assembled exactly from the partial
// outputs and their log-sum-exp values:
//   L = ln(e^a + e^b),  out = e^(a - L) o_pp + e^(b - L) o_ps.
// HBM-bound elementwise pass: 2 x fp32 [Np, H, d] read, out patch rows written in the
// layer dtype. Each thread handles 8 consecutive elements of one (token, head) row;
// a grid-stride loop over a grid sized to the SM count.
#include <cmath>

#include "common.cuh"

namespace bsa {
namespace {

template <typename T>
__global__ void __launch_bounds__(256)
merge_kernel(Geo g, const float* __restrict__ o_pp, const float* __restrict__ lse_pp,
             const float* __restrict__ o_ps, const float* __restrict__ lse_ps, T* __restrict__ out) {
    const size_t per_row = (size_t)g.H * g.d / 8;     // 8-element groups per token
    const size_t total = (size_t)g.Np * per_row;
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < total;
         x += (size_t)gridDim.x * blockDim.x) {
        const int p = (int)(x / per_row);
        const int e0 = (int)(x - (size_t)p * per_row) * 8;
        const int h = e0 / g.d;
        const float a = __ldg(lse_pp + (size_t)h * g.Np + p);
        const float b = __ldg(lse_ps + (size_t)h * g.Np + p);
        const float mx = fmaxf(a, b);
        float wa = 0.f, wb = 0.f;
        if (mx != -INFINITY) {
            const float L = mx + log1pf(expf(-fabsf(a - b)));
            wa = expf(a - L);
            wb = expf(b - L);
        }
        const size_t src = (size_t)p * g.H * g.d + e0;
        const float4* pa = reinterpret_cast<const float4*>(o_pp + src);
        const float4* pb = reinterpret_cast<const float4*>(o_ps + src);
        float r[8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float4 va = __ldg(pa + u);
            const float4 vb = __ldg(pb + u);
            r[4 * u + 0] = wa * va.x + wb * vb.x;
            r[4 * u + 1] = wa * va.y + wb * vb.y;
            r[4 * u + 2] = wa * va.z + wb * vb.z;
            r[4 * u + 3] = wa * va.w + wb * vb.w;
        }
        T* dst = out + (size_t)patch_row(g, p) * g.H * g.d + e0;
        if constexpr (sizeof(T) == 2) {
            Vec16<T>::store(dst, r);
        } else {
            Vec16<T>::store(dst, r);
            Vec16<T>::store(dst + 4, r + 4);
        }
    }
}

__global__ void fill_kernel(float* __restrict__ p, size_t n, float value) {
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < n; x += (size_t)gridDim.x * blockDim.x)
        p[x] = value;
}

}  // namespace

cudaError_t launch_fill(float* p, size_t n, float value, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    fill_kernel<<<num_sms() * 4, 256, 0, st>>>(p, n, value);
    return cudaGetLastError();
}

cudaError_t launch_merge(const Geo& g, bsa_dtype dt, const float* o_pp, const float* lse_pp,
                         const float* o_ps, const float* lse_ps, void* out, cudaStream_t st) {
    const int grid = num_sms() * 8;
    if (dt == BSA_BF16)
        merge_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(g, o_pp, lse_pp, o_ps, lse_ps,
                                                          static_cast<__nv_bfloat16*>(out));
    else
        merge_kernel<float><<<grid, 256, 0, st>>>(g, o_pp, lse_pp, o_ps, lse_ps, static_cast<float*>(out));
    return cudaGetLastError();
}

}  // namespace bsa
