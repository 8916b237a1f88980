// Frame-wise dense attention on the tensor cores: every token attends over the T tokens of its
// own frame (the frame half of the aggregator that alternates frame-wise and global attention,
// "Block-Sparse Global Attention for Efficient Multi-View Geometry Transformers", 研究背景与动机;
// "SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction Transformers", 图2).
//
// Input: the per-frame packing of pack.cu (frame_layout): per head and frame, the frame's T
// tokens padded with zero rows to t_pad = ceil(T / 128) 128 rows; Q, K bf16, V fp16.
//
// The CTA is the one of the global layer's attention (tc kernel of attn_tc.cu): TMA producer
// warp, one MMA thread (S = Q K^T into TMEM columns [0,128), O += P V with P in [128,192) and O
// in [192,256)), four softmax warps with one query row per thread, two CTAs per SM. A frame has
// only ceil(T / 128) key tiles (7 at T = 782), so one query tile is short work; the CTAs here are
// persistent: each walks query tiles (head, frame, tile) with a stride of the grid, and the
// barriers run on across tiles (a running tile count gives each wait its phase), so the
// producer loads the next item's Q and first K/V tiles while the current item's last tiles and
// epilogue run. Barrier protocol, per key tile U (running count) and item I:
//   kv_full / kv_empty  ring of NS stages of K and V tiles;
//   q_full / q_empty    the Q tile of item I; the MMA thread commits q_empty after the
//                       item's last QK^T, the producer waits on it before the next Q load;
//   s_full, s_free, p_full, o_done   as in the global layer's kernel;
//   o_final             committed after the item's last P.V; the softmax waits on it, reads O,
//                       writes the rows, and only then arrives on p_full of the next item's
//                       first tile, so the next item's first P.V (which overwrites O) follows.
// A frame's last key tile holds T mod 128 keys (14 at T = 782): its QK^T runs at N = the keys
// rounded up to 16, its P.V over the 16-key steps that hold keys, and the softmax skips the
// exponentials and P stores of the 32-key chunks past T.
// Every wait is bounded; a timeout is reported through the status word.
#include <cuda.h>

#include <cmath>

#include "common.cuh"
#include "sm100.cuh"
#include "tc_layout.cuh"
#include "tma_map.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kFThreads = 192;
constexpr int kFStages = 3;
constexpr uint32_t kFTmemCols = 256, kFColS = 0, kFColP = 128, kFColO = 192;
constexpr float kFScaleLog2 = 0.18033688011112042f;   // log2(e) / sqrt(64)
constexpr float kFRescale = 8.0f;
constexpr uint32_t kFTile = 128 * 128;                // bytes of a 128-row tile of 64 two-byte elements
constexpr uint32_t kFOffQ = 0, kFOffK = kFTile, kFOffV = kFOffK + kFStages * kFTile,
                   kFOffCtl = kFOffV + kFStages * kFTile;

struct FCtl {
    uint64_t q_full, q_empty;
    uint64_t kv_full[kFStages], kv_empty[kFStages];
    uint64_t s_full, s_free, p_full, o_done, o_final, drain;
    uint32_t tmem_base;
    int abort;
};

struct FParams {
    Geo g;
    int t_pad;        // packed rows per (head, frame)
    int f_tiles;      // key (and query) tiles per frame
    int items;        // H * F * f_tiles query tiles
    __nv_bfloat16* out;
    int32_t* status;
};

__device__ __forceinline__ bool fwarp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status));
}

__global__ void __launch_bounds__(kFThreads, 2)
frame_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FParams prm) {
    extern __shared__ __align__(1024) uint8_t smem[];
    FCtl& ctl = *reinterpret_cast<FCtl*>(smem + kFOffCtl);
    const Geo& g = prm.g;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &ctl.abort;
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) record_error(prm.status, BSA_ERR_DEVICE_BOUNDS);
        return;
    }
    const int nt = prm.f_tiles;
    if (threadIdx.x == 0) {
        mbar_init(&ctl.q_full, 1);
        mbar_init(&ctl.q_empty, 1);
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(&ctl.kv_full[s], 1);
            mbar_init(&ctl.kv_empty[s], 1);
        }
        mbar_init(&ctl.s_full, 1);
        mbar_init(&ctl.s_free, 4);
        mbar_init(&ctl.p_full, 4);
        mbar_init(&ctl.o_done, 1);
        mbar_init(&ctl.o_final, 1);
        mbar_init(&ctl.drain, 1);
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, kFTmemCols);
        tmem_relinquish();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    int issued = 0;   // K/V tiles whose loads the producer issued (running count)
    int q_loads = 0;  // Q tiles the producer issued

    if (warp == 0) {
        // ============================================================ TMA producer
        if (lane == 0) {
            int U = 0, I = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < prm.items; item += gridDim.x, ++I) {
                const int hf = item / nt, ft = item - hf * nt;   // (head, frame), query tile
                const int row0 = hf * prm.t_pad;
                if (I > 0 && !mbar_wait(&ctl.q_empty, (I - 1) & 1, abort, prm.status)) break;
                mbar_arrive_expect_tx(&ctl.q_full, kFTile);
                tma_load_2d(smem + kFOffQ, &tm_q, &ctl.q_full, 0, row0 + ft * 128);
                q_loads = I + 1;
                for (int u = 0; u < nt; ++u, ++U) {
                    const int st = U % kFStages;
                    if (U >= kFStages && !mbar_wait(&ctl.kv_empty[st], ((U / kFStages) - 1) & 1, abort, prm.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ctl.kv_full[st], 2 * kFTile);
                    tma_load_2d(smem + kFOffK + st * kFTile, &tm_k, &ctl.kv_full[st], 0, row0 + u * 128);
                    tma_load_2d(smem + kFOffV + st * kFTile, &tm_v, &ctl.kv_full[st], 0, row0 + u * 128);
                    issued = U + 1;
                }
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_pv = idesc_f16(128, 64, 0u, true);
            const uint32_t q_base = smem_u32(smem + kFOffQ);
            // QK^T of key tile u of an item, over its keys rounded up to 16 (a frame's last
            // tile holds T mod 128 keys)
            auto issue_qk = [&](int U, int u) -> bool {
                const int st = U % kFStages;
                if (!mbar_wait(&ctl.kv_full[st], (U / kFStages) & 1, abort, prm.status)) return false;
                tc_fence_after();
                const uint32_t k_base = smem_u32(smem + kFOffK + st * kFTile);
                const int n16 = (min(128, g.T - u * 128) + 15) & ~15;
                const uint32_t idesc_qk = idesc_f16(128, n16, 1u, false);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kFColS, sdesc_sw128(q_base + 32 * ks, 16, 1024), sdesc_sw128(k_base + 32 * ks, 16, 1024),
                           idesc_qk, ks > 0 ? 1u : 0u);
                mma_commit(&ctl.s_full);
                return true;
            };
            int U = 0, I = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < prm.items; item += gridDim.x, ++I) {
                if (!mbar_wait(&ctl.q_full, I & 1, abort, prm.status)) break;
                // the previous item's last S has been read by the softmax
                if (I > 0 && !mbar_wait(&ctl.s_free, (U - 1) & 1, abort, prm.status)) break;
                if (!(ok = issue_qk(U, 0))) break;
                if (nt == 1) mma_commit(&ctl.q_empty);
                for (int u = 0; u < nt; ++u) {
                    const int Uu = U + u;
                    if (u + 1 < nt) {
                        if (!mbar_wait(&ctl.s_free, Uu & 1, abort, prm.status)) { ok = false; break; }
                        if (!(ok = issue_qk(Uu + 1, u + 1))) break;
                        if (u + 2 == nt) mma_commit(&ctl.q_empty);   // the item's last QK^T is issued
                    }
                    if (!mbar_wait(&ctl.p_full, Uu & 1, abort, prm.status)) { ok = false; break; }
                    tc_fence_after();
                    const int st = Uu % kFStages;
                    const uint32_t v_base = smem_u32(smem + kFOffV + st * kFTile);
                    const int k16 = (min(128, g.T - u * 128) + 15) / 16;   // 16-key steps holding keys
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        if (ks < k16)
                            mma_ts(tmem + kFColO, tmem + kFColP + 8 * ks, sdesc_sw128(v_base + 2048 * ks, 0, 1024),
                                   idesc_pv, (u > 0 || ks > 0) ? 1u : 0u);
                    mma_commit(&ctl.kv_empty[st]);
                    mma_commit(&ctl.o_done);
                    if (u == nt - 1) mma_commit(&ctl.o_final);
                }
                U += nt;
            }
        }
    } else {
        // ============================================================ softmax + epilogue
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        int U = 0, I = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < prm.items; item += gridDim.x, ++I) {
            const int hf = item / nt, ft = item - hf * nt;
            const int h = hf / g.F, f = hf - h * g.F;
            float m_ref = -INFINITY, l = 0.f;
            for (int u = 0; u < nt; ++u) {
                const int Uu = U + u;
                const int nvalid = min(128, g.T - u * 128);
                const bool full = nvalid == 128;
                if (!fwarp_wait(&ctl.s_full, Uu & 1, abort, prm.status)) { ok = false; break; }
                tc_fence_after();
                uint32_t s[128];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tmem_ld32(lane_base + kFColS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.s_free);
                float mt = -INFINITY;
                if (full) {
                    float acc[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = __uint_as_float(s[i]);
#pragma unroll
                    for (int c = 8; c < 128; c += 2)
                        acc[(c / 2) & 7] = max3f(acc[(c / 2) & 7], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
                    mt = max3f(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c < nvalid) mt = fmaxf(mt, __uint_as_float(s[c]));
                }
                const float mt2 = mt * kFScaleLog2;
                const bool need = mt2 > m_ref + kFRescale;
                const bool corr = need && m_ref != -INFINITY;
                const float new_ref = need ? mt2 : m_ref;
                const float factor = corr ? ex2_approx(m_ref - new_ref) : 1.f;
                m_ref = new_ref;
                float rs = 0.f;
                if (full) {
                    float2 r2[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) r2[i] = make_float2(0.f, 0.f);
                    const float2 scale2 = make_float2(kFScaleLog2, kFScaleLog2);
                    const float2 shift2 = make_float2(-m_ref, -m_ref);
#pragma unroll
                    for (int c = 0; c < 128; c += 2) {
                        const int i = c / 2;
                        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                                    scale2, shift2);
                        const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        r2[i & 3] = __fadd2_rn(r2[i & 3], pr);
                        s[i] = pack_half2(pr.x, pr.y);
                    }
                    rs = ((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y));
                } else {
                    // the frame's last tile: chunks of 32 keys, those past T skipped (warp-uniform)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (32 * k < nvalid) {
#pragma unroll
                            for (int c = 32 * k; c < 32 * k + 32; c += 2) {
                                const float p0 =
                                    c < nvalid ? ex2_approx(fmaf(__uint_as_float(s[c]), kFScaleLog2, -m_ref)) : 0.f;
                                const float p1 =
                                    c + 1 < nvalid ? ex2_approx(fmaf(__uint_as_float(s[c + 1]), kFScaleLog2, -m_ref))
                                                   : 0.f;
                                rs += p0 + p1;
                                s[c / 2] = pack_half2(p0, p1);
                            }
                        } else {
#pragma unroll
                            for (int c = 32 * k; c < 32 * k + 32; c += 2) s[c / 2] = 0u;
                        }
                    }
                }
                l = l * factor + rs;
                // P.V of the item's previous tile must be done before O is rescaled or P is
                // overwritten (for the first tile, the previous item's o_final wait covered it)
                if (u > 0 && !fwarp_wait(&ctl.o_done, (Uu - 1) & 1, abort, prm.status)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, corr)) {
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + kFColO + 32 * a, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
                        tmem_st32(lane_base + kFColO + 32 * a, o);
                    }
                }
#pragma unroll
                for (int c = 0; c < 2; ++c)   // P.V reads only the 16-key steps that hold keys
                    if (64 * c < nvalid)
                        tmem_st32(lane_base + kFColP + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&s[32 * c]));
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.p_full);
            }
            if (!ok) break;
            // epilogue of the item: O / l for the frame's rows
            if (!fwarp_wait(&ctl.o_final, I & 1, abort, prm.status)) { ok = false; break; }
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int r = ft * 128 + row;
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                uint32_t v[32];
                tmem_ld32(lane_base + kFColO + 32 * a, v);
                tmem_wait_ld();
                if (r < g.T) {
                    float o[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(v[c]) * inv;
                    __nv_bfloat16* dst = prm.out + ((size_t)f * g.T + r) * g.H * 64 + (size_t)h * 64 + 32 * a;
#pragma unroll
                    for (int c = 0; c < 32; c += 8) Vec16<__nv_bfloat16>::store(dst + c, o + c);
                }
            }
            tc_fence_before();
            U += nt;
        }
    }

    // ------------------------------------------------------------------ teardown
    __syncthreads();
    if (ctl.abort) {
        if (warp == 0 && lane == 0) {
            volatile int never = 0;
            if (q_loads > 0) mbar_wait(&ctl.q_full, (q_loads - 1) & 1, &never, prm.status, 50000000ull);
            for (int u = max(0, issued - kFStages); u < issued; ++u)
                mbar_wait(&ctl.kv_full[u % kFStages], (u / kFStages) & 1, &never, prm.status, 50000000ull);
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
        tmem_dealloc(tmem, kFTmemCols);
    }
}

}  // namespace

// Frame-wise attention over the per-frame packing in ws; writes every row of out (bf16).
cudaError_t launch_attn_frame(const Geo& g, const void* ws, void* out, int32_t* status, cudaStream_t st) {
    const FrameLayout fl = frame_layout(g);
    const uint8_t* base = static_cast<const uint8_t*>(ws);
    FParams prm;
    prm.g = g;
    prm.t_pad = fl.t_pad;
    prm.f_tiles = fl.t_pad / 128;
    prm.items = g.H * g.F * prm.f_tiles;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.status = status;
    const uint64_t rows = (uint64_t)g.H * g.F * fl.t_pad;
    CUtensorMap q, k, v;
    if (!make_tile_map(&q, base + fl.qf, rows, 64, 128, false) || !make_tile_map(&k, base + fl.kf, rows, 64, 128, false) ||
        !make_tile_map(&v, base + fl.vf, rows, 64, 128, true))
        return cudaErrorInvalidValue;
    if (prm.items == 0) return cudaSuccess;
    const size_t smem = kFOffCtl + (sizeof(FCtl) + 15) / 16 * 16;
    cudaError_t e = cudaFuncSetAttribute(frame_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = prm.items < 2 * num_sms() ? prm.items : 2 * num_sms();
    frame_attn_kernel<<<grid, kFThreads, smem, st>>>(q, k, v, prm);
    return cudaGetLastError();
}

}  // namespace bsa
