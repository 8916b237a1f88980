// Tensor-core attention for the bf16 layer on B200 (sm_100a): tcgen05 MMA with TMEM
// accumulators, TMA tile loads, fp32 online softmax. It covers the three attention pieces
// of "Block-Sparse Global Attention for Efficient Multi-View Geometry Transformers":
//   MODE_SPARSE        patch query tile over the kept key blocks of its query blocks
//                      (关键设计 1, Eq. (2); masked entries are excluded) -> o_pp, lse_pp
//   MODE_PATCH_SPECIAL patch query tile over every special key (关键设计 3)  -> o_ps, lse_ps
//   MODE_SPECIAL_ALL   special query tile over every key (关键设计 3)       -> out (bf16)
//
// Inputs come from the packed workspace (pack.cu): per head, 64-wide rows of 128 bytes,
// so each query tile (128 rows) and each key tile (BKV = b rows, or 128) is one 2D TMA box
// with the 128-byte swizzle that the MMA descriptors expect.
//
// One CTA per (query tile, head), 6 warps:
//   warp 0      TMA producer: Q once, then K/V tiles into an NS-stage ring;
//   warp 1      MMA issuer (one thread): S = Q K^T into one of two TMEM S buffers, and
//               O += P V with P read from TMEM (fp16, written over its S buffer);
//   warps 2..5  softmax, one query row per thread (TMEM lane = row): row max, lazy
//               rescale of O (only when the running max grows by more than 2^8),
//               p = 2^(s log2(e)/sqrt(d) - m) in fp32, P rounded to fp16 into TMEM,
//               then the epilogue O / l and the log-sum-exp.
// For b = 64 a 128-row query tile holds two query blocks; it walks the union of their
// kept blocks, and each row ignores the key blocks its own query block did not keep.
// Every mbarrier wait is bounded; a timeout is reported through the status word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"
#include "tc_layout.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0;
constexpr uint32_t kColS1 = 128;
constexpr uint32_t kColO = 256;
constexpr float kScaleLog2 = 0.18033688011112042f;   // log2(e) / sqrt(64)
constexpr float kRescale = 8.0f;                     // lazy-rescale threshold (log2 units)
constexpr float kLn2 = 0.69314718055994531f;
constexpr int kThreads = 192;

enum { MODE_SPARSE = 0, MODE_PATCH_SPECIAL = 1, MODE_SPECIAL_ALL = 2 };

struct TcParams {
    Geo g;
    PackedLayout pl;
    const uint16_t* kv_idx;
    const int32_t* kv_cnt;
    float* o_part;
    float* lse_part;
    __nv_bfloat16* out;
    int32_t* status;
};

template <int BKV>
struct Cfg {
    static constexpr int NS = BKV == 128 ? 4 : 8;   // K/V stages
    static constexpr int QB = 128 / BKV;            // query blocks per 128-row query tile
    static constexpr uint32_t kTileBytes = BKV * 128;
    static constexpr uint32_t kOffQ = 0;
    static constexpr uint32_t kOffK = kOffQ + 128 * 128;
    static constexpr uint32_t kOffV = kOffK + NS * kTileBytes;
    static constexpr uint32_t kOffCtl = kOffV + NS * kTileBytes;
};

template <int NS>
struct Ctl {
    uint64_t q_full;
    uint64_t kv_full[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done;
    uint64_t o_final;
    uint64_t drain;
    int meta_nvalid[NS];
    uint32_t meta_member[NS];
    uint32_t tmem_base;
    int n_tiles;
    int abort;
};

template <int BKV>
constexpr size_t smem_bytes() {
    return Cfg<BKV>::kOffCtl + ((sizeof(Ctl<Cfg<BKV>::NS>) + 15) / 16 * 16) +
           (size_t)Cfg<BKV>::QB * (BSA_MAX_BLOCKS / 32) * 4 + 1024;
}

// Lane 0 waits, the whole warp gets the same answer (keeps .sync.aligned tcgen05 ops uniform).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status,
                                          int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, abort, status);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
    volatile int never = 0;
    return mbar_wait(bar, parity, &never, status, 50000000ull);
}

template <int MODE, int BKV>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k0,
               const __grid_constant__ CUtensorMap tm_v0, const __grid_constant__ CUtensorMap tm_k1,
               const __grid_constant__ CUtensorMap tm_v1, const TcParams prm) {
    using C = Cfg<BKV>;
    constexpr int NS = C::NS;
    constexpr int QB = C::QB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl<NS>& ctl = *reinterpret_cast<Ctl<NS>*>(smem + C::kOffCtl);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + C::kOffCtl + (sizeof(Ctl<NS>) + 15) / 16 * 16);
    const Geo& g = prm.g;
    const PackedLayout& pl = prm.pl;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int h = blockIdx.x % g.H;
    const int tq = blockIdx.x / g.H;
    volatile int* abort = &ctl.abort;
    const int words = (g.B + 31) / 32;

    // ------------------------------------------------------------------ setup
    if (threadIdx.x == 0) {
        mbar_init(&ctl.q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&ctl.kv_full[s], 1);
            mbar_init(&ctl.kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.s_full[b], 1);
            mbar_init(&ctl.p_full[b], 4);
        }
        mbar_init(&ctl.o_done, 1);
        mbar_init(&ctl.o_final, 1);
        mbar_init(&ctl.drain, 1);
        ctl.n_tiles = 0;
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k0);
        tma_prefetch(&tm_v0);
        if (MODE == MODE_SPECIAL_ALL) {
            tma_prefetch(&tm_k1);
            tma_prefetch(&tm_v1);
        }
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (MODE == MODE_SPARSE) {
        for (int x = threadIdx.x; x < QB * words; x += kThreads) bits[x] = 0u;
        __syncthreads();
        for (int qb = 0; qb < QB; ++qb) {
            const int i = tq * QB + qb;
            if (i >= g.B) break;
            int cnt = prm.kv_cnt[(size_t)h * g.B + i];
            if (cnt > g.B) {
                if (threadIdx.x == 0) record_error(prm.status, BSA_ERR_DEVICE_BOUNDS);
                cnt = g.B;
            }
            const uint16_t* list = prm.kv_idx + ((size_t)h * g.B + i) * g.B;
            for (int t = threadIdx.x; t < cnt; t += kThreads) {
                const int j = list[t];
                if (j >= g.B) record_error(prm.status, BSA_ERR_DEVICE_BOUNDS);
                else atomicOr(&bits[qb * words + (j >> 5)], 1u << (j & 31));
            }
        }
        __syncthreads();
        int local = 0;
        for (int w = threadIdx.x; w < words; w += kThreads) {
            uint32_t u = 0;
            for (int qb = 0; qb < QB; ++qb) u |= bits[qb * words + w];
            local += __popc(u);
        }
        if (local) atomicAdd(&ctl.n_tiles, local);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const int ns_tiles = (g.Ns + 127) / 128;
    const int n = MODE == MODE_SPARSE ? ctl.n_tiles
                : MODE == MODE_PATCH_SPECIAL ? ns_tiles
                : ns_tiles + (g.Np + 127) / 128;
    int issued = 0;   // K/V tiles whose loads the producer issued

    if (warp == 0) {
        // ============================================================ TMA producer
        if (lane == 0) {
            const int q_row0 = MODE == MODE_SPECIAL_ALL ? h * pl.ns_pad + tq * 128 : h * pl.np_pad + tq * 128;
            mbar_arrive_expect_tx(&ctl.q_full, 128 * 128);
            tma_load_2d(smem + C::kOffQ, &tm_q, &ctl.q_full, 0, q_row0);
            int w = 0;
            uint32_t cur = 0;
            if (MODE == MODE_SPARSE && words > 0)
                for (int qb = 0; qb < QB; ++qb) cur |= bits[qb * words];
            for (int t = 0; t < n; ++t) {
                const int stage = t % NS;
                if (t >= NS && !mbar_wait(&ctl.kv_empty[stage], ((t / NS) - 1) & 1, abort, prm.status)) break;
                int row0, nvalid;
                uint32_t member = 1u;
                const CUtensorMap* mk = &tm_k0;
                const CUtensorMap* mv = &tm_v0;
                if (MODE == MODE_SPARSE) {
                    while (cur == 0u && w + 1 < words) {
                        ++w;
                        for (int qb = 0; qb < QB; ++qb) cur |= bits[qb * words + w];
                    }
                    if (cur == 0u) break;
                    const int bit = __ffs(cur) - 1;
                    cur &= cur - 1u;
                    const int j = w * 32 + bit;
                    member = 0u;
                    for (int qb = 0; qb < QB; ++qb) member |= ((bits[qb * words + w] >> bit) & 1u) << qb;
                    row0 = h * pl.np_pad + j * BKV;
                    nvalid = min(BKV, g.Np - j * BKV);
                } else if (MODE == MODE_PATCH_SPECIAL || t < ns_tiles) {
                    row0 = h * pl.ns_pad + t * 128;
                    nvalid = min(128, g.Ns - t * 128);
                } else {
                    const int u = t - ns_tiles;
                    row0 = h * pl.np_pad + u * 128;
                    nvalid = min(128, g.Np - u * 128);
                    mk = &tm_k1;
                    mv = &tm_v1;
                }
                ctl.meta_nvalid[stage] = nvalid;
                ctl.meta_member[stage] = member;
                mbar_arrive_expect_tx(&ctl.kv_full[stage], 2 * C::kTileBytes);
                tma_load_2d(smem + C::kOffK + stage * C::kTileBytes, mk, &ctl.kv_full[stage], 0, row0);
                tma_load_2d(smem + C::kOffV + stage * C::kTileBytes, mv, &ctl.kv_full[stage], 0, row0);
                issued = t + 1;
            }
            if (n == 0) drain_wait(&ctl.q_full, 0, prm.status);   // no MMA will consume Q
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0 && n > 0 && mbar_wait(&ctl.q_full, 0, abort, prm.status)) {
            constexpr uint32_t idesc_qk = idesc_f16(128, BKV, 1u, false);
            constexpr uint32_t idesc_pv = idesc_f16(128, 64, 0u, true);
            const uint32_t q_base = smem_u32(smem + C::kOffQ);
            auto issue_qk = [&](int t) -> bool {
                const int stage = t % NS;
                if (!mbar_wait(&ctl.kv_full[stage], (t / NS) & 1, abort, prm.status)) return false;
                tc_fence_after();
                const uint32_t sbuf = tmem + ((t & 1) ? kColS1 : kColS0);
                const uint32_t k_base = smem_u32(smem + C::kOffK + stage * C::kTileBytes);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(sbuf, sdesc_sw128(q_base + 32 * ks, 16, 1024), sdesc_sw128(k_base + 32 * ks, 16, 1024),
                           idesc_qk, ks > 0 ? 1u : 0u);
                mma_commit(&ctl.s_full[t & 1]);
                return true;
            };
            bool ok = issue_qk(0);
            if (ok && n > 1) ok = issue_qk(1);
            for (int t = 0; ok && t < n; ++t) {
                if (!mbar_wait(&ctl.p_full[t & 1], (t >> 1) & 1, abort, prm.status)) break;
                tc_fence_after();
                const int stage = t % NS;
                const uint32_t sbuf = tmem + ((t & 1) ? kColS1 : kColS0);
                const uint32_t v_base = smem_u32(smem + C::kOffV + stage * C::kTileBytes);
#pragma unroll
                for (int ks = 0; ks < BKV / 16; ++ks)
                    mma_ts(tmem + kColO, sbuf + 8 * ks, sdesc_sw128(v_base + 2048 * ks, 0, 1024), idesc_pv,
                           (t > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&ctl.kv_empty[stage]);
                mma_commit(&ctl.o_done);
                if (t == n - 1) mma_commit(&ctl.o_final);
                if (t + 2 < n) {
                    if (!mbar_wait(&ctl.o_done, t & 1, abort, prm.status)) break;   // P_t consumed
                    ok = issue_qk(t + 2);
                }
            }
        }
    } else {
        // ============================================================ softmax
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int row_qb = row / BKV;
        float m_ref = -INFINITY;
        float l = 0.f;
        bool ok = true;
        for (int t = 0; t < n; ++t) {
            const int stage = t % NS;
            if (!warp_wait(&ctl.kv_full[stage], (t / NS) & 1, abort, prm.status, lane)) { ok = false; break; }
            const int nvalid = ctl.meta_nvalid[stage];
            const bool member = ((ctl.meta_member[stage] >> row_qb) & 1u) != 0u;
            if (!warp_wait(&ctl.s_full[t & 1], (t >> 1) & 1, abort, prm.status, lane)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sbuf = lane_base + ((t & 1) ? kColS1 : kColS0);
            uint32_t s[BKV];
#pragma unroll
            for (int c = 0; c < BKV / 32; ++c)
                tmem_ld32(sbuf + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
            tmem_wait_ld();
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < BKV; ++c)
                if (member && c < nvalid) mt = fmaxf(mt, __uint_as_float(s[c]));
            const float mt2 = mt * kScaleLog2;
            const bool need = mt2 > m_ref + kRescale;
            const bool corr = need && m_ref != -INFINITY;
            const float new_ref = need ? mt2 : m_ref;
            if (__any_sync(0xffffffffu, corr)) {
                const float factor = corr ? ex2_approx(m_ref - new_ref) : 1.f;
                if (t > 0 && !warp_wait(&ctl.o_done, (t - 1) & 1, abort, prm.status, lane)) { ok = false; break; }
                tc_fence_after();
                uint32_t o[2][32];
                tmem_ld32(lane_base + kColO, o[0]);
                tmem_ld32(lane_base + kColO + 32, o[1]);
                tmem_wait_ld();
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[a][c] = __float_as_uint(__uint_as_float(o[a][c]) * factor);
                tmem_st32(lane_base + kColO, o[0]);
                tmem_st32(lane_base + kColO + 32, o[1]);
                tmem_wait_st();
                l *= factor;
            }
            m_ref = new_ref;
            uint32_t pk[BKV / 2];
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < BKV; c += 2) {
                const bool v0 = member && c < nvalid;
                const bool v1 = member && c + 1 < nvalid;
                const float p0 = v0 ? ex2_approx(fmaf(__uint_as_float(s[c]), kScaleLog2, -m_ref)) : 0.f;
                const float p1 = v1 ? ex2_approx(fmaf(__uint_as_float(s[c + 1]), kScaleLog2, -m_ref)) : 0.f;
                rs += p0 + p1;
                const __half2 hp = __floats2half2_rn(p0, p1);
                pk[c / 2] = *reinterpret_cast<const uint32_t*>(&hp);
            }
            l += rs;
#pragma unroll
            for (int c = 0; c < BKV / 64; ++c)
                tmem_st32(sbuf + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32 * c]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.p_full[t & 1]);
        }
        // ------------------------------------------------------------ epilogue
        float o[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) o[c] = 0.f;
        // A parity wait only tells apart phases within one of the barrier's current phase.
        // Here o_done may still be two phases behind (tile n-1 done by this warp, P.V of
        // tile n-2 still running), so the epilogue waits on its own single-phase barrier.
        if (ok && n > 0 && warp_wait(&ctl.o_final, 0, abort, prm.status, lane)) {
            tc_fence_after();
            uint32_t r[2][32];
            tmem_ld32(lane_base + kColO, r[0]);
            tmem_ld32(lane_base + kColO + 32, r[1]);
            tmem_wait_ld();
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                o[c] = __uint_as_float(r[0][c]) * inv;
                o[32 + c] = __uint_as_float(r[1][c]) * inv;
            }
        } else if (n > 0) {
            l = 0.f;   // aborted: report an empty row
        }
        const float lse = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
        if (MODE == MODE_SPECIAL_ALL) {
            const int ts = tq * 128 + row;
            if (ts < g.Ns) {
                __nv_bfloat16* dst = prm.out + (size_t)special_row(g, ts) * g.H * 64 + (size_t)h * 64;
#pragma unroll
                for (int c = 0; c < 64; c += 8) Vec16<__nv_bfloat16>::store(dst + c, o + c);
            }
        } else {
            const int p = tq * 128 + row;
            if (p < g.Np) {
                float* dst = prm.o_part + ((size_t)p * g.H + h) * 64;
#pragma unroll
                for (int c = 0; c < 64; c += 4) Vec16<float>::store(dst + c, o + c);
                prm.lse_part[(size_t)h * g.Np + p] = lse;
            }
        }
    }

    // ------------------------------------------------------------------ teardown
    __syncthreads();
    if (ctl.abort) {
        // let in-flight copies and MMAs land before the shared and tensor memory go away
        if (warp == 0 && lane == 0)
            for (int t = max(0, issued - NS); t < issued; ++t)
                drain_wait(&ctl.kv_full[t % NS], (t / NS) & 1, prm.status);
        if (warp == 1 && lane == 0) {
            mma_commit(&ctl.drain);
            drain_wait(&ctl.drain, 0, prm.status);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D map over `rows` rows of 64 two-byte elements (128-byte pitch), box of box_rows rows.
bool make_map(CUtensorMap* tm, const void* base, uint64_t rows, uint32_t box_rows, bool fp16) {
    auto enc = get_encode();
    if (enc == nullptr || rows == 0) return false;
    cuuint64_t dims[2] = {64, rows};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(tm, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int BKV>
cudaError_t launch_mode(const TcParams& prm, const CUtensorMap& q, const CUtensorMap& k0, const CUtensorMap& v0,
                        const CUtensorMap& k1, const CUtensorMap& v1, int q_tiles, cudaStream_t st) {
    const size_t smem = smem_bytes<BKV>();
    auto kern = attn_tc_kernel<MODE, BKV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<q_tiles * prm.g.H, kThreads, smem, st>>>(q, k0, v0, k1, v1, prm);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const Geo& g, int mode, const void* ws, const uint16_t* kv_idx,
                           const int32_t* kv_cnt, float* o_part, float* lse_part, void* out,
                           int32_t* status, cudaStream_t st) {
    const PackedLayout pl = packed_layout(g);
    const uint8_t* base = static_cast<const uint8_t*>(ws);
    TcParams prm;
    prm.g = g;
    prm.pl = pl;
    prm.kv_idx = kv_idx;
    prm.kv_cnt = kv_cnt;
    prm.o_part = o_part;
    prm.lse_part = lse_part;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.status = status;
    const uint64_t prow = (uint64_t)g.H * pl.np_pad;
    const uint64_t srow = (uint64_t)g.H * pl.ns_pad;
    CUtensorMap q, k0, v0, k1, v1;
    if (mode == MODE_SPARSE) {
        if (!make_map(&q, base + pl.qp, prow, 128, false) || !make_map(&k0, base + pl.kp, prow, g.b, false) ||
            !make_map(&v0, base + pl.vp, prow, g.b, true))
            return cudaErrorInvalidValue;
        const int q_tiles = pl.np_pad / 128;
        return g.b == 128 ? launch_mode<MODE_SPARSE, 128>(prm, q, k0, v0, k0, v0, q_tiles, st)
                          : launch_mode<MODE_SPARSE, 64>(prm, q, k0, v0, k0, v0, q_tiles, st);
    }
    if (g.Ns == 0) return cudaSuccess;
    if (!make_map(&k0, base + pl.ks, srow, 128, false) || !make_map(&v0, base + pl.vs, srow, 128, true))
        return cudaErrorInvalidValue;
    if (mode == MODE_PATCH_SPECIAL) {
        if (!make_map(&q, base + pl.qp, prow, 128, false)) return cudaErrorInvalidValue;
        return launch_mode<MODE_PATCH_SPECIAL, 128>(prm, q, k0, v0, k0, v0, pl.np_pad / 128, st);
    }
    if (!make_map(&q, base + pl.qs, srow, 128, false) || !make_map(&k1, base + pl.kp, prow, 128, false) ||
        !make_map(&v1, base + pl.vp, prow, 128, true))
        return cudaErrorInvalidValue;
    return launch_mode<MODE_SPECIAL_ALL, 128>(prm, q, k0, v0, k1, v1, pl.ns_pad / 128, st);
}

}  // namespace bsa
