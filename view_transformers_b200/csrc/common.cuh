// Shared device-side definitions of the block-sparse attention library (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "bsa.h"

namespace bsa {

// Geometry of one layer, derived once on the host (see bsa.h for the token layout).
struct Geo {
    int F, T, S, H, d, b;
    int P;   // patch tokens per frame
    int N;   // tokens
    int Np;  // patch tokens
    int Ns;  // special tokens
    int B;   // blocks
};

// Row of patch token p of the concatenated patch sequence X_p.
__device__ __forceinline__ int patch_row(const Geo& g, int p) {
    const int f = p / g.P;
    return f * g.T + g.S + (p - f * g.P);
}

// Row of special token t (0 <= t < Ns): the first S tokens of every frame.
__device__ __forceinline__ int special_row(const Geo& g, int t) {
    const int f = t / g.S;
    return f * g.T + (t - f * g.S);
}

// First device-side error wins; later ones are dropped.
__device__ __forceinline__ void record_error(int32_t* status, int32_t code) {
    if (status != nullptr) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// 16-byte vector of T unpacked to floats.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int n = 4;
    __device__ __forceinline__ static void load(const float* p, float* out) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    __device__ __forceinline__ static void store(float* p, const float* in) {
        *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* in) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

}  // namespace bsa

// Internal launchers (defined in the .cu files, called by the C ABI in abi.cu).
namespace bsa {
cudaError_t launch_pool(const Geo& g, bsa_dtype dt, const void* q, const void* k, float* pq,
                        float* pk, cudaStream_t st);
struct MaskParams {
    int k[BSA_MAX_HEADS];
    double tau;
};
cudaError_t launch_mask(const Geo& g, const MaskParams& mp, const float* pq, const float* pk,
                        uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                        int32_t* status, cudaStream_t st);
cudaError_t launch_attn_simt(const Geo& g, bsa_dtype dt, int mode, const void* q, const void* k,
                             const void* v, const uint16_t* kv_idx, const int32_t* kv_cnt,
                             float* o_part, float* lse_part, void* out, int32_t* status,
                             cudaStream_t st);
cudaError_t launch_merge(const Geo& g, bsa_dtype dt, const float* o_pp, const float* lse_pp,
                         const float* o_ps, const float* lse_ps, void* out, cudaStream_t st);
cudaError_t launch_fill(float* p, size_t n, float value, cudaStream_t st);
cudaError_t launch_wait_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t st);
int num_sms();
}  // namespace bsa
