// fp32 CUDA-core attention for the float32 layout (small layers), covering the three
// attention pieces of the layer ("Block-Sparse Global Attention for Efficient Multi-View
// Geometry Transformers"):
//   mode 0  patch query block i over the patch keys of its kept blocks (Eq. (2))
//           -> o_pp [Np, H, d] fp32, lse_pp [H, Np]
//   mode 1  patch query block i over the special keys (关键设计 3, X_p -> X_s)
//           -> o_ps, lse_ps
//   mode 2  special queries over every token (关键设计 3, X_s -> all) -> out (final)
// Online softmax over key chunks of up to 64 rows, accurate expf/logf, fp32 throughout:
// the float32 path must stay within 1e-5 of the fp64 oracle, which tensor-core tf32
// inputs would not.
#include <cfloat>

#include "common.cuh"

namespace bsa {
namespace {

constexpr int kQ = 64;        // query rows per tile
constexpr int kC = 64;        // key rows per chunk
constexpr int kD = 64;        // head dim
constexpr int kStride = kD + 1;
constexpr int kThreads = 256; // 4 threads per query row

struct Smem {
    float q[kQ][kStride];
    float k[kC][kStride];
    float v[kC][kStride];
    float p[kQ][kC + 1];
    int krow[kC];
    int qrow[kQ];
};

template <typename T>
__device__ void load_rows(float (*dst)[kStride], const int* rows, int n, const T* src, int h,
                          const Geo& g) {
    const size_t rs = (size_t)g.H * g.d;
    for (int x = threadIdx.x; x < kC * kD; x += kThreads) {
        const int r = x / kD, c = x % kD;
        dst[r][c] = r < n ? to_f32(src[(size_t)rows[r] * rs + (size_t)h * g.d + c]) : 0.f;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(Geo g, int mode, const T* __restrict__ q, const T* __restrict__ k,
                 const T* __restrict__ v, const uint16_t* __restrict__ kv_idx,
                 const int32_t* __restrict__ kv_cnt, float* __restrict__ o_part,
                 float* __restrict__ lse_part, T* __restrict__ out, int32_t* status) {
    extern __shared__ __align__(16) unsigned char raw[];
    Smem& sm = *reinterpret_cast<Smem*>(raw);
    const int h = blockIdx.y;
    const int r = threadIdx.x / 4;      // query row within the tile
    const int part = threadIdx.x % 4;   // key/dim quarter owned by this thread
    const float scale = rsqrtf((float)g.d);

    // query rows of this CTA: patch block i (modes 0, 1) or special tile (mode 2)
    int q_lo, q_hi;
    if (mode == 2) {
        q_lo = blockIdx.x * kQ;
        q_hi = min(q_lo + kQ, g.Ns);
    } else {
        q_lo = blockIdx.x * g.b;
        q_hi = min(q_lo + g.b, g.Np);
    }
    for (int t0 = q_lo; t0 < q_hi; t0 += kQ) {
        const int nq = min(kQ, q_hi - t0);
        __syncthreads();
        for (int x = threadIdx.x; x < kQ; x += kThreads)
            sm.qrow[x] = x < nq ? (mode == 2 ? special_row(g, t0 + x) : patch_row(g, t0 + x)) : 0;
        __syncthreads();
        load_rows(sm.q, sm.qrow, nq, q, h, g);

        float m = -FLT_MAX;   // running max of scaled scores (no key seen yet)
        float l = 0.f;        // running sum of exp(score - m)
        float o[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) o[x] = 0.f;

        // enumerate key chunks
        const int nblk = mode == 0 ? kv_cnt[(size_t)h * g.B + blockIdx.x] : 1;
        for (int t = 0; t < nblk; ++t) {
            int k_lo, k_hi;
            if (mode == 0) {
                const int j = kv_idx[((size_t)h * g.B + blockIdx.x) * g.B + t];
                if (j < 0 || j >= g.B) {
                    record_error(status, BSA_ERR_DEVICE_BOUNDS);
                    continue;
                }
                k_lo = j * g.b;
                k_hi = min(k_lo + g.b, g.Np);
            } else if (mode == 1) {
                k_lo = 0;
                k_hi = g.Ns;
            } else {
                k_lo = 0;
                k_hi = g.N;
            }
            for (int c0 = k_lo; c0 < k_hi; c0 += kC) {
                const int nk = min(kC, k_hi - c0);
                __syncthreads();
                for (int x = threadIdx.x; x < kC; x += kThreads)
                    sm.krow[x] = x < nk ? (mode == 0 ? patch_row(g, c0 + x)
                                           : mode == 1 ? special_row(g, c0 + x) : c0 + x) : 0;
                __syncthreads();
                load_rows(sm.k, sm.krow, nk, k, h, g);
                load_rows(sm.v, sm.krow, nk, v, h, g);
                __syncthreads();
                // scores of row r against keys part, part+4, ...
                float s[16];
                float cmax = -FLT_MAX;
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int c = part + 4 * x;
                    float acc = 0.f;
                    if (c < nk) {
#pragma unroll 16
                        for (int dd = 0; dd < kD; ++dd) acc = fmaf(sm.q[r][dd], sm.k[c][dd], acc);
                        acc *= scale;
                        cmax = fmaxf(cmax, acc);
                    }
                    s[x] = acc;
                }
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
                const float mnew = fmaxf(m, cmax);
                const float alpha = expf(m - mnew);
                float psum = 0.f;
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int c = part + 4 * x;
                    const float p = c < nk ? expf(s[x] - mnew) : 0.f;
                    psum += p;
                    sm.p[r][c] = p;
                }
                psum += __shfl_xor_sync(0xffffffffu, psum, 1);
                psum += __shfl_xor_sync(0xffffffffu, psum, 2);
                l = l * alpha + psum;
                m = mnew;
                __syncwarp();
#pragma unroll
                for (int x = 0; x < 16; ++x) o[x] *= alpha;
                for (int c = 0; c < nk; ++c) {
                    const float p = sm.p[r][c];
#pragma unroll
                    for (int x = 0; x < 16; ++x) o[x] = fmaf(p, sm.v[c][part * 16 + x], o[x]);
                }
            }
        }
        // epilogue
        if (r < nq) {
            const bool empty = l <= 0.f;
            const float inv = empty ? 0.f : 1.f / l;
            const int t = t0 + r;
            if (mode == 2) {
                T* dst = out + (size_t)sm.qrow[r] * g.H * g.d + (size_t)h * g.d + part * 16;
#pragma unroll
                for (int x = 0; x < 16; ++x) dst[x] = from_f32<T>(o[x] * inv);
            } else {
                float* dst = o_part + ((size_t)t * g.H + h) * g.d + part * 16;
#pragma unroll
                for (int x = 0; x < 16; ++x) dst[x] = o[x] * inv;
                if (part == 0) lse_part[(size_t)h * g.Np + t] = empty ? -INFINITY : m + logf(l);
            }
        }
    }
}

}  // namespace

cudaError_t launch_attn_simt(const Geo& g, bsa_dtype dt, int mode, const void* q, const void* k,
                             const void* v, const uint16_t* kv_idx, const int32_t* kv_cnt,
                             float* o_part, float* lse_part, void* out, int32_t* status,
                             cudaStream_t st) {
    const int tiles = mode == 2 ? (g.Ns + kQ - 1) / kQ : g.B;
    if (tiles == 0) return cudaSuccess;
    const dim3 grid(tiles, g.H);
    const size_t smem = sizeof(Smem);
    if (dt == BSA_F32) {
        cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attn_simt_kernel<float><<<grid, kThreads, smem, st>>>(
            g, mode, static_cast<const float*>(q), static_cast<const float*>(k),
            static_cast<const float*>(v), kv_idx, kv_cnt, o_part, lse_part, static_cast<float*>(out), status);
    } else {
        cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attn_simt_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(
            g, mode, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), kv_idx, kv_cnt, o_part, lse_part,
            static_cast<__nv_bfloat16*>(out), status);
    }
    return cudaGetLastError();
}

}  // namespace bsa
