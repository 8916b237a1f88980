// Projections on either side of the attention layer: y = x W^T + b with bf16 inputs, fp32
// accumulation and bf16 outputs. The pages place the global attention between the QKV and
// output projections of a multi-head attention block ("Block-Sparse Global Attention for
// Efficient Multi-View Geometry Transformers", 研究背景与动机: the alternating frame / global
// attention aggregator; "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
// Transformers", 图2).
//
// One persistent CTA per SM walks 128 x 256 output tiles (m-major: consecutive tiles share
// their A rows, and W stays in L2). K advances in steps of 64 elements, one 128-byte swizzle
// atom, through a 4-stage TMA ring (48 KB per stage). 6 warps:
//   warp 0      TMA producer (A box 64 x 128, B box 64 x 256; rows past the end read zeros);
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma M = 128, N = 256, K = 16 per step into
//               one of two 256-column TMEM accumulators;
//   warps 2..5  epilogue, one output row per thread (TMEM lane = row): tcgen05.ld 32 columns
//               at a time, + bias, round to bf16, 64-byte stores.
// With two accumulators the epilogue of tile t runs while the MMAs of tile t+1 proceed.
// Barriers: full[s]/empty[s] (ring), acc_full[b] (commit after a tile's last MMA),
// acc_empty[b] (4 epilogue warps). Every wait is bounded (status word on timeout).
//
// Outputs: column n of the product goes to out[n / split] at [row, n % split] (row stride
// `split`), so the QKV projection writes Q, K and V as three [N, H, d] tensors in one pass.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_map.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr uint32_t kABytes = kBM * kBK * 2, kBBytes = kBN * kBK * 2;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kGemmThreads = 192;

struct GemmCtl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct GemmParams {
    int M, N, K;
    int split;                       // columns per output tensor
    __nv_bfloat16* out[3];
    const float* bias;               // [N] or null
    int32_t* status;
};

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const GemmParams prm) {
    extern __shared__ __align__(1024) uint8_t smem[];
    GemmCtl& ctl = *reinterpret_cast<GemmCtl*>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &ctl.abort;
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) record_error(prm.status, BSA_ERR_DEVICE_BOUNDS);
        return;
    }
    const int m_tiles = (prm.M + kBM - 1) / kBM, n_tiles = (prm.N + kBN - 1) / kBN;
    const int tiles = m_tiles * n_tiles, ksteps = prm.K / kBK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], 4);
        }
        mbar_init(&ctl.drain, 1);
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_a);
        tma_prefetch(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, 512);
        tmem_relinquish();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    int issued = 0;   // ring loads the producer issued

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * kBN;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !mbar_wait(&ctl.empty[s], ((it / kStages) - 1) & 1, abort, prm.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(&ctl.full[s], kStageBytes);
                    tma_load_2d(st, &tm_a, &ctl.full[s], ks * kBK, m0);
                    tma_load_2d(st + kABytes, &tm_b, &ctl.full[s], ks * kBK, n0);
                    issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(kBM, kBN, 1u, false);
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                if (lt >= 2 && !mbar_wait(&ctl.acc_empty[b], ((lt >> 1) - 1) & 1, abort, prm.status)) break;
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(b * kBN);
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&ctl.full[s], (it / kStages) & 1, abort, prm.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * kStageBytes);
                    const uint32_t b_base = a_base + kABytes;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        mma_ss(acc, sdesc_sw128(a_base + 32 * k, 16, 1024), sdesc_sw128(b_base + 32 * k, 16, 1024),
                               idesc, (ks > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&ctl.empty[s]);
                }
                if (ok) mma_commit(&ctl.acc_full[b]);
            }
        }
    } else {
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&ctl.acc_full[b], (lt >> 1) & 1, abort, prm.status))) break;
            tc_fence_after();
            const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * kBN;
            const int row = m0 + r;
            const uint32_t acc = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * kBN);
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                const int n = n0 + c * 32;
                if (n >= prm.N) break;   // warp-uniform
                uint32_t v[32];
                tmem_ld32(acc + 32 * c, v);
                tmem_wait_ld();
                if (row < prm.M) {
                    float x[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(v[i]);
                    if (prm.bias != nullptr) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 bb = __ldg(reinterpret_cast<const float4*>(prm.bias + n + i));
                            x[i] += bb.x; x[i + 1] += bb.y; x[i + 2] += bb.z; x[i + 3] += bb.w;
                        }
                    }
                    const int which = n / prm.split;
                    __nv_bfloat16* dst = prm.out[which] + (size_t)row * prm.split + (n - which * prm.split);
#pragma unroll
                    for (int i = 0; i < 32; i += 8) Vec16<__nv_bfloat16>::store(dst + i, x + i);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.acc_empty[b]);
        }
    }

    __syncthreads();
    if (ctl.abort) {
        if (warp == 0 && lane == 0)
            for (int u = max(0, issued - kStages); u < issued; ++u) {
                volatile int never = 0;
                mbar_wait(&ctl.full[u % kStages], (u / kStages) & 1, &never, prm.status, 50000000ull);
            }
        if (warp == 1 && lane == 0) {
            volatile int never = 0;
            mma_commit(&ctl.drain);
            mbar_wait(&ctl.drain, 0, &never, prm.status, 50000000ull);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------
// The same product on CTA pairs: a cluster of two CTAs (the two SMs of a TPC) computes a
// 256 x 256 output tile with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16). Each CTA
// loads its own 128 rows of A and its half (128 rows) of the B tile, so a K-step moves 32 KB
// into each SM for 512 MMA cycles (64 bytes per clock, against 96 for a 128 x 256 tile on one
// SM), and holds its 128 rows of D in its own TMEM (two 256-column accumulators).
// Roles (same warps in both CTAs):
//   warp 0      TMA producer of this CTA's half of each stage; the even CTA also posts the
//               stage's expected bytes (both halves) on its own full[s], which both CTAs'
//               copies complete;
//   warp 1      MMA issuer in the even CTA only (one thread); its commits arrive on the
//               barriers of both CTAs (empty[s], acc_full[b]);
//   warps 2..5  epilogue of this CTA's 128 rows; acc_empty[b] of the even CTA counts the
//               four epilogue warps of both CTAs.
// Both CTAs walk the same pair tiles (clusters strided over the tiles), so every barrier
// phase lines up. Every wait is bounded.
constexpr int kPStages = 6;
constexpr uint32_t kPABytes = 128 * kBK * 2, kPBBytes = 128 * kBK * 2;
constexpr uint32_t kPStageBytes = kPABytes + kPBBytes;

struct PairCtl {
    uint64_t full[kPStages];
    uint64_t empty[kPStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int issued;   // loads issued by this CTA's producer
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const GemmParams prm) {
    extern __shared__ __align__(1024) uint8_t smem[];
    PairCtl& ctl = *reinterpret_cast<PairCtl*>(smem + kPStages * kPStageBytes);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &ctl.abort;
    // identical in both CTAs of the pair (same kernel, same layout), so both leave together
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) record_error(prm.status, BSA_ERR_DEVICE_BOUNDS);
        return;
    }
    const uint32_t rank = cluster_ctarank();
    const bool even = rank == 0;
    const int pair = (int)cluster_id_x(), npairs = (int)ncluster_x();
    const int m_tiles = (prm.M + 255) / 256, n_tiles = (prm.N + 255) / 256;
    const int tiles = m_tiles * n_tiles, ksteps = prm.K / kBK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], 8);
        }
        mbar_init(&ctl.drain, 1);
        ctl.abort = 0;
        ctl.issued = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_a);
        tma_prefetch(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl.tmem_base, 512);
        tmem_relinquish_pair();
    }
    __syncthreads();
    cluster_sync();   // both CTAs' barriers exist before either signals the other's
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    // the even CTA's barriers, as seen from this CTA
    const uint32_t full0 = mapa_shared(smem_u32(&ctl.full[0]), 0);
    const uint32_t acc_empty0 = mapa_shared(smem_u32(&ctl.acc_empty[0]), 0);

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = pair; ok && t < tiles; t += npairs) {
                const int m0 = (t / n_tiles) * 256 + (int)rank * 128;
                const int n0 = (t % n_tiles) * 256 + (int)rank * 128;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kPStages;
                    if (it >= kPStages && !mbar_wait(&ctl.empty[s], ((it / kPStages) - 1) & 1, abort, prm.status)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(&ctl.full[s], 2 * kPStageBytes);
                    uint8_t* st = smem + s * kPStageBytes;
                    const uint32_t bar = full0 + (uint32_t)(s * sizeof(uint64_t));
                    tma_load_2d_pair(st, &tm_a, bar, ks * kBK, m0);
                    tma_load_2d_pair(st + kPABytes, &tm_b, bar, ks * kBK, n0);
                    ctl.issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && even) {
            constexpr uint32_t idesc = idesc_f16(256, 256, 1u, false);
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = pair; ok && t < tiles; t += npairs, ++lt) {
                const int b = lt & 1;
                if (lt >= 2 && !mbar_wait(&ctl.acc_empty[b], ((lt >> 1) - 1) & 1, abort, prm.status)) break;
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(b * 256);
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kPStages;
                    if (!mbar_wait(&ctl.full[s], (it / kPStages) & 1, abort, prm.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * kPStageBytes);
                    const uint32_t b_base = a_base + kPABytes;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        mma_ss_pair(acc, sdesc_sw128(a_base + 32 * k, 16, 1024), sdesc_sw128(b_base + 32 * k, 16, 1024),
                                    idesc, (ks > 0 || k > 0) ? 1u : 0u);
                    mma_commit_pair_both(&ctl.empty[s]);
                }
                if (ok) mma_commit_pair_both(&ctl.acc_full[b]);
            }
        }
    } else {
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        int lt = 0;
        for (int t = pair; t < tiles; t += npairs, ++lt) {
            const int b = lt & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&ctl.acc_full[b], (lt >> 1) & 1, abort, prm.status))) break;
            tc_fence_after();
            const int row = (t / n_tiles) * 256 + (int)rank * 128 + r;
            const int n0 = (t % n_tiles) * 256;
            const uint32_t acc = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * 256);
#pragma unroll 1
            for (int c = 0; c < 256 / 32; ++c) {
                const int n = n0 + c * 32;
                if (n >= prm.N) break;   // warp-uniform
                uint32_t v[32];
                tmem_ld32(acc + 32 * c, v);
                tmem_wait_ld();
                if (row < prm.M) {
                    float x[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(v[i]);
                    if (prm.bias != nullptr) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 bb = __ldg(reinterpret_cast<const float4*>(prm.bias + n + i));
                            x[i] += bb.x; x[i + 1] += bb.y; x[i + 2] += bb.z; x[i + 3] += bb.w;
                        }
                    }
                    const int which = n / prm.split;
                    __nv_bfloat16* dst = prm.out[which] + (size_t)row * prm.split + (n - which * prm.split);
#pragma unroll
                    for (int i = 0; i < 32; i += 8) Vec16<__nv_bfloat16>::store(dst + i, x + i);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0 + (uint32_t)(b * sizeof(uint64_t)));
        }
    }

    __syncthreads();
    cluster_sync();   // both CTAs have left their loops; the peer's load count is final
    if (even && warp == 0 && lane == 0) {
        // after an abort, let the copies in flight (both CTAs' halves complete on this CTA's
        // full barriers) land before shared memory goes away; bounded waits
        const int peer_issued = ld_shared_cluster_s32(mapa_shared(smem_u32(&ctl.issued), 1));
        const int issued = max(ctl.issued, peer_issued);
        if (ctl.abort || peer_issued != ctl.issued)
            for (int u = max(0, issued - kPStages); u < issued; ++u) {
                volatile int never = 0;
                mbar_wait(&ctl.full[u % kPStages], (u / kPStages) & 1, &never, prm.status, 50000000ull);
            }
    }
    if (even && warp == 1 && lane == 0 && ctl.abort) {
        volatile int never = 0;
        mma_commit_pair(&ctl.drain);
        mbar_wait(&ctl.drain, 0, &never, prm.status, 50000000ull);
    }
    __syncthreads();
    cluster_sync();   // no MMA of the pair still writes either CTA's TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

constexpr size_t kPairSmem = kPStages * kPStageBytes + sizeof(PairCtl);

// Clusters of two gemm_pair_kernel CTAs the current device holds at once (0: use the
// single-CTA kernel). Queried once per device.
int pair_clusters() {
    static int cache[64];
    static std::once_flag once[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::call_once(once[dev], [dev] {
        int n = 0;
        if (cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmem) ==
            cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * num_sms(), 1, 1);
            cfg.blockDim = dim3(kGemmThreads, 1, 1);
            cfg.dynamicSmemBytes = kPairSmem;
            if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &cfg) != cudaSuccess) n = 0;
        }
        cudaGetLastError();   // a refused query leaves no sticky error behind
        cache[dev] = n;
    });
    return cache[dev];
}

}  // namespace

// y = a b^T + bias: a [M, K], b [N, K] (row-major bf16), outputs as described above.
// Needs K % 64 == 0, N % 32 == 0, split % 32 == 0, N <= 3 split, 16-byte aligned pointers.
cudaError_t launch_gemm_bf16(int M, int N, int K, const void* a, const void* b, const float* bias,
                             void* const out[3], int split, int32_t* status, cudaStream_t st) {
    if (M <= 0 || N <= 0 || K <= 0 || K % kBK != 0 || N % 32 != 0 || split % 32 != 0 || N > 3 * split)
        return cudaErrorInvalidValue;
    CUtensorMap ta, tb;
    if (!make_tile_map(&ta, a, (uint64_t)M, (uint64_t)K, kBM, false) || !make_tile_map(&tb, b, (uint64_t)N, (uint64_t)K, kBN, false))
        return cudaErrorInvalidValue;
    GemmParams prm;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.split = split;
    for (int i = 0; i < 3; ++i) prm.out[i] = static_cast<__nv_bfloat16*>(out[i]);
    prm.bias = bias;
    prm.status = status;
    // CTA pairs: as many clusters as the device holds at once (one CTA per SM)
    const int pairs = pair_clusters();
    if (pairs > 0) {
        CUtensorMap tbp;
        if (!make_tile_map(&tbp, b, (uint64_t)N, (uint64_t)K, 128, false)) return cudaErrorInvalidValue;
        const long long tiles = (long long)((M + 255) / 256) * ((N + 255) / 256);
        const int grid = 2 * (int)(tiles < pairs ? tiles : pairs);
        gemm_pair_kernel<<<grid, kGemmThreads, kPairSmem, st>>>(ta, tbp, prm);
        return cudaGetLastError();
    }
    const size_t smem = kStages * kStageBytes + sizeof(GemmCtl);
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    gemm_bf16_kernel<<<grid, kGemmThreads, smem, st>>>(ta, tb, prm);
    return cudaGetLastError();
}

}  // namespace bsa
