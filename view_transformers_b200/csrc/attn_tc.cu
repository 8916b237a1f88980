// Tensor-core attention for the bf16 layer on B200 (sm_100a): tcgen05 MMA with TMEM
// accumulators, TMA tile loads, fp32 online softmax. It covers the attention pieces of
// "Block-Sparse Global Attention for Efficient Multi-View Geometry Transformers":
//   MODE_SPARSE        patch query tile over the kept key blocks of its query blocks
//                      (关键设计 1, Eq. (2); masked entries are excluded) -> o_pp, lse_pp
//   MODE_PATCH_SPECIAL patch query tile over every special key (关键设计 3)  -> o_ps, lse_ps
//   MODE_SPECIAL_ALL   special query tile over one chunk of all keys (关键设计 3) -> split
//                      partials in the workspace, combined by special_combine_kernel
//   MODE_FUSED         patch query tile over the special keys and the kept key blocks in
//                      one online softmax: steps 4, 5(ii) and the merge in one pass -> out
//
// Inputs come from the packed workspace (pack.cu): per head, 64-wide rows of 128 bytes,
// so a query tile (128 rows) is one 2D TMA box with the 128-byte swizzle that the MMA
// descriptors expect, and a 128-key tile is one box of b = 128 rows or two of b = 64.
//
// One CTA per work item, two CTAs per SM (112 KB of shared memory and 256 TMEM columns
// each, so the softmax of one CTA overlaps the tensor-core work of the other). 6 warps:
//   warp 0      TMA producer: Q once, then K/V tiles into an NS-stage ring;
//   warp 1      MMA issuer (one thread): S = Q K^T (TMEM columns [0,128)), then
//               O += P V with P (fp16) read from TMEM columns [128,192), O in [192,256);
//               the next S is computed as soon as the softmax has read the current one;
//   warps 2..5  softmax, one query row per thread (TMEM lane = row): row max, lazy
//               rescale of O (only when the running max grows by more than 2^8),
//               p = 2^(s log2(e)/sqrt(d) - m) in fp32, P rounded to fp16 into TMEM,
//               then the epilogue O / l and the log-sum-exp.
// For b = 64 a 128-row query tile holds two query blocks; it walks the union of their
// kept blocks, two per 128-key tile. A warp's 32 rows share a query block, so the softmax
// branches per warp on which of the tile's two key blocks that query block kept: both (all
// 128 columns), one (its 64 columns, P = 0 for the other) or neither (P = 0); only tiles
// with a ragged kept block go column by column.
//
// Barrier protocol (u = tile index of the CTA). A parity wait only tells apart phases
// within one phase of the barrier's current one; every wait below has that property:
//   kv_full[s]/kv_empty[s]  TMA ring; the producer refills a stage after P.V of its tile.
//            For b = 64 the softmax also waits on kv_full to read the tile's extent and
//            membership, which the producer stores per stage;
//   s_full   QK^T of tile u done (commit; also implies every earlier MMA is done);
//   s_free   all 4 softmax warps have S_u in registers (count 4) -> QK^T of tile u+1;
//   p_full   all 4 softmax warps wrote P_u (count 4) -> P.V of tile u;
//   o_done   P.V of tile u done (commit). The softmax waits o_done(u-1) before writing
//            P_u or rescaling O: at tile u it has seen s_full(u), so P.V of tile u-2 is
//            done and o_done is at most one phase behind;
//   o_final  single phase, committed after the last P.V: the epilogue waits on it.
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

constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColO = 192;
constexpr float kScaleLog2 = 0.18033688011112042f;   // log2(e) / sqrt(64)
constexpr float kRescale = 8.0f;                     // lazy-rescale threshold (log2 units)
constexpr float kLn2 = 0.69314718055994531f;
constexpr int kThreads = 192;

enum { MODE_SPARSE = 0, MODE_PATCH_SPECIAL = 1, MODE_SPECIAL_ALL = 2, MODE_FUSED = 3 };

struct TcParams {
    Geo g;
    PackedLayout pl;
    const uint16_t* kv_idx;
    const int32_t* kv_cnt;
    float* o_part;
    float* lse_part;
    __nv_bfloat16* out;
    float* spart;
    float* slse;
    int32_t* status;
    int q_tiles;   // query tiles per head
};

// BKV is the block size b (64 or 128). Query and key tiles are always 128 rows: a key tile
// holds one block of 128 keys or two kept blocks of 64 (not necessarily adjacent), so that
// QK^T runs at N = 128 and each tile's fixed costs cover 128 keys.
template <int BKV>
struct Cfg {
    static constexpr int NS = 3;                    // K/V stages
    static constexpr int QB = 128 / BKV;            // query blocks per 128-row query tile
    static constexpr int KB = 128 / BKV;            // key blocks per 128-key tile
    static constexpr uint32_t kTileBytes = 128 * 128;
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
    uint64_t s_full;
    uint64_t s_free;
    uint64_t p_full;
    uint64_t o_done;
    uint64_t o_final;
    uint64_t drain;
    int meta_nvalid[NS];     // tile extents for the softmax when it does not compute them: row
    uint32_t meta_member[NS];   // counts of the key blocks (8 bits each) and their membership bits
    uint32_t tmem_base;
    int n_tiles;
    int abort;
    int head;
};

// The key tiles of one CTA, in order: one key range of special and patch tiles
// (MODE_SPECIAL_ALL), every special tile (MODE_PATCH_SPECIAL), or, for the fused and sparse
// modes, the special tiles (fused only) followed by the kept blocks of the CTA's query blocks
// (the union of their masks, ascending), KB blocks per tile. The producer runs it, and for
// b = 128 the softmax warps run the arithmetic part of their own copy, so they learn a tile's
// extent without a barrier. A tile with fewer than KB kept blocks left loads its missing
// block from a row past the end of the packed array, which reads zeros.
template <int MODE, int BKV>
struct TileWalk {
    static constexpr int QB = 128 / BKV;
    static constexpr int KB = 128 / BKV;
    struct Tile {
        int row0[KB];      // first packed row of each key block
        int nvalid[KB];    // rows of each key block that hold keys (0 for a missing block)
        uint32_t member;   // bit k * QB + qb: query block qb of the tile kept key block k
        bool special;      // tile of special keys
    };
    const uint32_t* bits;
    int words;
    int w = 0;
    uint32_t cur = 0u;
    __device__ __forceinline__ TileWalk(const uint32_t* b, int nw) : bits(b), words(nw) {
        if ((MODE == MODE_SPARSE || MODE == MODE_FUSED) && nw > 0)
            for (int qb = 0; qb < QB; ++qb) cur |= bits[qb * nw];
    }
    // Tile u (called for u = 0, 1, ... in order). False only if the union has no further
    // block, which cannot happen for u below the CTA's tile count.
    __device__ __forceinline__ bool next(int u, const Geo& g, const PackedLayout& pl, int h, int sp_tiles,
                                         int t_begin, Tile& t) {
        t.member = (1u << (KB * QB)) - 1u;
        if (MODE == MODE_SPECIAL_ALL) {
            const int x = t_begin + u;
            t.special = x < sp_tiles;
            const int base = t.special ? x * 128 : (x - sp_tiles) * 128;
            t.row0[0] = (t.special ? h * pl.ns_pad : h * pl.np_pad) + base;
            t.nvalid[0] = min(128, (t.special ? g.Ns : g.Np) - base);
            return true;
        }
        if (MODE == MODE_PATCH_SPECIAL || (MODE == MODE_FUSED && u < sp_tiles)) {
            t.special = true;
#pragma unroll
            for (int k = 0; k < KB; ++k) {
                t.row0[k] = h * pl.ns_pad + u * 128 + k * BKV;
                t.nvalid[k] = max(0, min(BKV, g.Ns - (u * 128 + k * BKV)));
            }
            return true;
        }
        t.special = false;
        t.member = 0u;
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            while (cur == 0u && w + 1 < words) {
                ++w;
                for (int qb = 0; qb < QB; ++qb) cur |= bits[qb * words + w];
            }
            if (cur == 0u) {
                if (k == 0) return false;
                t.row0[k] = g.H * pl.np_pad;   // past the end: zeros
                t.nvalid[k] = 0;
                continue;
            }
            const int bit = __ffs(cur) - 1;
            cur &= cur - 1u;
            const int j = w * 32 + bit;
            for (int qb = 0; qb < QB; ++qb) t.member |= ((bits[qb * words + w] >> bit) & 1u) << (k * QB + qb);
            t.row0[k] = h * pl.np_pad + j * BKV;
            t.nvalid[k] = min(BKV, g.Np - j * BKV);
        }
        return true;
    }
};

template <int BKV>
size_t smem_bytes(int num_blocks) {
    const size_t words = (size_t)(num_blocks + 31) / 32;
    return Cfg<BKV>::kOffCtl + (sizeof(Ctl<Cfg<BKV>::NS>) + 15) / 16 * 16 + Cfg<BKV>::QB * words * 4;
}

// Every lane polls and the warp votes, so no divergent branch has to reconverge (a lane-0
// wait followed by a shuffle costs about 2.5x as much on B200, even on a completed phase).
// The vote keeps the .sync.aligned tcgen05 ops that follow uniform. A lane cannot miss the
// phase: each barrier a softmax warp waits on moves to its next phase only after that warp
// arrives on s_free or p_full.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status));
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
    volatile int never = 0;
    return mbar_wait(bar, parity, &never, status, 50000000ull);
}

template <int MODE, int BKV>
__global__ void __launch_bounds__(kThreads, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ka,
               const __grid_constant__ CUtensorMap tm_va, const __grid_constant__ CUtensorMap tm_kb,
               const __grid_constant__ CUtensorMap tm_vb, const TcParams prm) {
    using C = Cfg<BKV>;
    constexpr int NS = C::NS;
    constexpr int QB = C::QB;
    constexpr int KB = C::KB;
    constexpr bool kUnion = MODE == MODE_SPARSE || MODE == MODE_FUSED;   // walks kept blocks
    // With one query block per tile (b = 128) a softmax warp computes each tile's extent
    // itself; with two (b = 64) it reads what the producer stored for the stage, after the
    // stage's kv_full barrier (walking the union mask per warp costs more than that wait).
    constexpr bool kLocalTiles = KB == 1;
    extern __shared__ __align__(1024) uint8_t smem[];
    Ctl<NS>& ctl = *reinterpret_cast<Ctl<NS>*>(smem + C::kOffCtl);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + C::kOffCtl + (sizeof(Ctl<NS>) + 15) / 16 * 16);
    const Geo& g = prm.g;
    const PackedLayout& pl = prm.pl;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    volatile int* abort = &ctl.abort;
    const int words = (g.B + 31) / 32;

    // tile swizzles assume a 1024-byte aligned base; refuse to run otherwise
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) record_error(prm.status, BSA_ERR_DEVICE_BOUNDS);
        return;
    }

    // work item: head-major order keeps one head's keys hot in L2
    int h, tq, split = 0;
    if (MODE == MODE_SPECIAL_ALL) {
        const int per_head = prm.q_tiles * pl.nsplit;
        h = blockIdx.x / per_head;
        const int r = blockIdx.x - h * per_head;
        tq = r / pl.nsplit;
        split = r - tq * pl.nsplit;
    } else {
        h = blockIdx.x / prm.q_tiles;
        tq = blockIdx.x - h * prm.q_tiles;
    }
    const int sp_tiles = (g.Ns + 127) / 128;       // special key tiles (128 rows)
    int t_begin = 0, t_end = 0;                    // MODE_SPECIAL_ALL key-tile range
    if (MODE == MODE_SPECIAL_ALL) {
        const int n_all = sp_tiles + pl.np_pad / 128;   // even split: sizes differ by at most one
        t_begin = (int)((long long)split * n_all / pl.nsplit);
        t_end = (int)((long long)(split + 1) * n_all / pl.nsplit);
    }

    // ------------------------------------------------------------------ setup
    if (threadIdx.x == 0) {
        mbar_init(&ctl.q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&ctl.kv_full[s], 1);
            mbar_init(&ctl.kv_empty[s], 1);
        }
        mbar_init(&ctl.s_full, 1);
        mbar_init(&ctl.s_free, 4);
        mbar_init(&ctl.p_full, 4);
        mbar_init(&ctl.o_done, 1);
        mbar_init(&ctl.o_final, 1);
        mbar_init(&ctl.drain, 1);
        ctl.n_tiles = 0;
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_ka);
        tma_prefetch(&tm_va);
        tma_prefetch(&tm_kb);
        tma_prefetch(&tm_vb);
    }
    if (warp == 1) {
        tmem_alloc(&ctl.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (kUnion) {
        // Heads in descending order of kept work (the kept-block counts of three query-block
        // rows): CTAs of the heaviest heads start first, so the last wave holds light ones.
        // Consecutive CTAs keep sharing a head (its keys stay hot in L2).
        if (warp == 0) {
            const bool sortable = g.H <= 32;
            int w = -1;
            if (sortable && lane < g.H) {
                const int32_t* c = prm.kv_cnt + (size_t)lane * g.B;
                w = min(c[0], g.B) + min(c[g.B / 2], g.B) + min(c[g.B - 1], g.B);
            }
            int r = 0;
            for (int u = 0; u < 32; ++u) {
                const int wu = __shfl_sync(0xffffffffu, w, u);
                if (u < g.H && (wu > w || (wu == w && u < lane))) ++r;
            }
            const unsigned m = __ballot_sync(0xffffffffu, sortable && lane < g.H && r == h);
            if (lane == 0) ctl.head = m ? __ffs(m) - 1 : h;
        }
        for (int x = threadIdx.x; x < QB * words; x += kThreads) bits[x] = 0u;
        __syncthreads();
        h = ctl.head;
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
    const int kept_tiles = (ctl.n_tiles + KB - 1) / KB;   // KB kept blocks per tile
    const int n = MODE == MODE_SPARSE ? kept_tiles
                : MODE == MODE_FUSED ? sp_tiles + kept_tiles
                : MODE == MODE_PATCH_SPECIAL ? sp_tiles
                : t_end - t_begin;
    int issued = 0;   // K/V tiles whose loads the producer issued

    if (warp == 0) {
        // ============================================================ TMA producer
        if (lane == 0) {
            const int q_row0 = MODE == MODE_SPECIAL_ALL ? h * pl.ns_pad + tq * 128 : h * pl.np_pad + tq * 128;
            mbar_arrive_expect_tx(&ctl.q_full, 128 * 128);
            tma_load_2d(smem + C::kOffQ, &tm_q, &ctl.q_full, 0, q_row0);
            TileWalk<MODE, BKV> walk(bits, words);
            for (int u = 0; u < n; ++u) {
                const int stage = u % NS;
                if (u >= NS && !mbar_wait(&ctl.kv_empty[stage], ((u / NS) - 1) & 1, abort, prm.status)) break;
                typename TileWalk<MODE, BKV>::Tile t;
                if (!walk.next(u, g, pl, h, sp_tiles, t_begin, t)) break;
                if (!kLocalTiles) {
                    int nv = 0;
#pragma unroll
                    for (int k = 0; k < KB; ++k) nv |= t.nvalid[k] << (8 * k);
                    ctl.meta_nvalid[stage] = nv;
                    ctl.meta_member[stage] = t.member;
                }
                mbar_arrive_expect_tx(&ctl.kv_full[stage], 2 * C::kTileBytes);
#pragma unroll
                for (int k = 0; k < KB; ++k) {   // block k fills rows [k * BKV, (k + 1) * BKV) of the stage
                    const uint32_t off = stage * C::kTileBytes + (uint32_t)k * BKV * 128;
                    tma_load_2d(smem + C::kOffK + off, t.special ? &tm_ka : &tm_kb, &ctl.kv_full[stage], 0,
                                t.row0[k]);
                    tma_load_2d(smem + C::kOffV + off, t.special ? &tm_va : &tm_vb, &ctl.kv_full[stage], 0,
                                t.row0[k]);
                }
                issued = u + 1;
            }
            if (n == 0) drain_wait(&ctl.q_full, 0, prm.status);   // no MMA will consume Q
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0 && n > 0 && mbar_wait(&ctl.q_full, 0, abort, prm.status)) {
            constexpr uint32_t idesc_qk = idesc_f16(128, 128, 1u, false);
            constexpr uint32_t idesc_pv = idesc_f16(128, 64, 0u, true);
            const uint32_t q_base = smem_u32(smem + C::kOffQ);
            auto issue_qk = [&](int u) -> bool {
                const int stage = u % NS;
                if (!mbar_wait(&ctl.kv_full[stage], (u / NS) & 1, abort, prm.status)) return false;
                tc_fence_after();
                const uint32_t k_base = smem_u32(smem + C::kOffK + stage * C::kTileBytes);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kColS, sdesc_sw128(q_base + 32 * ks, 16, 1024),
                           sdesc_sw128(k_base + 32 * ks, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
                mma_commit(&ctl.s_full);
                return true;
            };
            bool ok = issue_qk(0);
            for (int u = 0; ok && u < n; ++u) {
                if (u + 1 < n) {
                    if (!mbar_wait(&ctl.s_free, u & 1, abort, prm.status)) break;   // S_u read
                    if (!issue_qk(u + 1)) break;
                }
                if (!mbar_wait(&ctl.p_full, u & 1, abort, prm.status)) break;
                tc_fence_after();
                const int stage = u % NS;
                const uint32_t v_base = smem_u32(smem + C::kOffV + stage * C::kTileBytes);
#pragma unroll
                for (int ks = 0; ks < 128 / 16; ++ks)
                    mma_ts(tmem + kColO, tmem + kColP + 8 * ks, sdesc_sw128(v_base + 2048 * ks, 0, 1024), idesc_pv,
                           (u > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&ctl.kv_empty[stage]);
                mma_commit(&ctl.o_done);
                if (u == n - 1) mma_commit(&ctl.o_final);
            }
        }
    } else {
        // ============================================================ softmax
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int row_qb = row / BKV;          // warp-uniform: a warp's 32 rows share a block
        float m_ref = -INFINITY;
        float l = 0.f;
        bool ok = true;
        // Tile extents as the producer's walk yields them. With one query block per tile the
        // kept blocks come in ascending order and each is a member, so only the last tile can
        // be the ragged last patch block; the special-key modes are plain arithmetic.
        const bool tail_kept = kLocalTiles && kUnion && g.B > 0 &&
                               ((bits[(g.B - 1) >> 5] >> ((g.B - 1) & 31)) & 1u) != 0u;
        const int tail_rows = g.Np - (g.B - 1) * BKV;
        TileWalk<MODE, BKV> walk(bits, 0);   // arithmetic modes only: no mask state
        constexpr int TC = 128;   // key columns per tile
        for (int u = 0; u < n; ++u) {
            int nvalid;
            uint32_t members = 1u;
            int nv1 = 0;            // b = 64: rows of the tile's second key block
            if (kLocalTiles && kUnion) {
                nvalid = MODE == MODE_FUSED && u < sp_tiles ? min(BKV, g.Ns - u * BKV)
                       : (u == n - 1 && tail_kept) ? tail_rows : BKV;
            } else if (kLocalTiles) {
                typename TileWalk<MODE, BKV>::Tile t;
                walk.next(u, g, pl, h, sp_tiles, t_begin, t);
                nvalid = t.nvalid[0];
            } else {
                const int stage = u % NS;
                if (!warp_wait(&ctl.kv_full[stage], (u / NS) & 1, abort, prm.status)) { ok = false; break; }
                const int packed = ctl.meta_nvalid[stage];
                nvalid = packed & 0xff;
                nv1 = (packed >> 8) & 0xff;
                members = ctl.meta_member[stage];
            }
            const bool member = ((members >> row_qb) & 1u) != 0u;
            bool full = member && nvalid == BKV;
            // b = 64: key block k of the tile is kept by this row's query block (mem1 for k = 1);
            // a tile is ragged when a kept block has fewer than 64 keys
            const bool mem1 = KB == 2 && ((members >> (QB + row_qb)) & 1u) != 0u;
            const bool ragged = KB == 2 && ((member && nvalid < BKV) || (mem1 && nv1 < BKV));
            if (KB == 2) full = !ragged;
            if (!warp_wait(&ctl.s_full, u & 1, abort, prm.status)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[TC];
#pragma unroll
            for (int c = 0; c < TC / 32; ++c)
                tmem_ld32(lane_base + kColS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.s_free);   // the next QK^T may overwrite S
            float mt = -INFINITY;
            if constexpr (KB == 2) {
                if (full) {   // both half maxima; a half this row's query block did not keep is dropped
                    float acc[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = __uint_as_float(s[(i & 3) + (i >> 2) * 64]);
#pragma unroll
                    for (int c = 4; c < 64; c += 2) {
                        acc[(c / 2) & 3] = max3f(acc[(c / 2) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
                        acc[4 + ((c / 2) & 3)] =
                            max3f(acc[4 + ((c / 2) & 3)], __uint_as_float(s[64 + c]), __uint_as_float(s[64 + c + 1]));
                    }
                    const float m0 = fmaxf(fmaxf(acc[0], acc[1]), fmaxf(acc[2], acc[3]));
                    const float m1 = fmaxf(fmaxf(acc[4], acc[5]), fmaxf(acc[6], acc[7]));
                    mt = fmaxf(member ? m0 : -INFINITY, mem1 ? m1 : -INFINITY);
                } else {
#pragma unroll
                    for (int c = 0; c < TC; ++c)
                        if (c < 64 ? (member && c < nvalid) : (mem1 && c - 64 < nv1))
                            mt = fmaxf(mt, __uint_as_float(s[c]));
                }
            } else {
            if (full) {   // 3-input max tree: short dependency chains
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = __uint_as_float(s[i]);
#pragma unroll
                for (int c = 8; c < BKV; c += 2)
                    acc[(c / 2) & 7] = max3f(acc[(c / 2) & 7], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
                mt = max3f(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
            } else if (member) {
#pragma unroll
                for (int c = 0; c < BKV; ++c)
                    if (c < nvalid) mt = fmaxf(mt, __uint_as_float(s[c]));
            }
            }
            const float mt2 = mt * kScaleLog2;
            const bool need = mt2 > m_ref + kRescale;
            const bool corr = need && m_ref != -INFINITY;
            const float new_ref = need ? mt2 : m_ref;
            const float factor = corr ? ex2_approx(m_ref - new_ref) : 1.f;
            m_ref = new_ref;
            // p in fp32, packed to fp16 pairs in place: pair i lands in s[i], after s[2i],
            // s[2i+1] were read
            float rs = 0.f;
            if constexpr (KB == 2) {
                if (full) {
                    // only the halves this row's query block kept (warp-uniform: a warp's 32
                    // rows share a query block); a half it did not keep gives P = 0
                    const float2 scale2 = make_float2(kScaleLog2, kScaleLog2);
                    const float2 shift2 = make_float2(-m_ref, -m_ref);
                    if (member && mem1) {
                        float2 r2[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) r2[i] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int c = 0; c < TC; c += 2) {
                            const int i = c / 2;
                            const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                                        scale2, shift2);
                            const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            r2[i & 3] = __fadd2_rn(r2[i & 3], pr);
                            s[i] = pack_half2(pr.x, pr.y);
                        }
                        rs = ((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y));
                    } else if (member) {   // first half only
                        float2 r2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                        for (int c = 0; c < 64; c += 2) {
                            const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                                        scale2, shift2);
                            const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            r2[(c / 2) & 1] = __fadd2_rn(r2[(c / 2) & 1], pr);
                            s[c / 2] = pack_half2(pr.x, pr.y);
                        }
#pragma unroll
                        for (int i = 32; i < 64; ++i) s[i] = 0u;
                        rs = (r2[0].x + r2[0].y) + (r2[1].x + r2[1].y);
                    } else if (mem1) {     // second half only
                        float2 r2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                        for (int c = 64; c < 128; c += 2) {
                            const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                                        scale2, shift2);
                            const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            r2[(c / 2) & 1] = __fadd2_rn(r2[(c / 2) & 1], pr);
                            s[c / 2] = pack_half2(pr.x, pr.y);
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) s[i] = 0u;
                        rs = (r2[0].x + r2[0].y) + (r2[1].x + r2[1].y);
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; ++i) s[i] = 0u;
                        rs = 0.f;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < TC; c += 2) {
                        const bool v0 = c < 64 ? (member && c < nvalid) : (mem1 && c - 64 < nv1);
                        const bool v1 = c + 1 < 64 ? (member && c + 1 < nvalid) : (mem1 && c + 1 - 64 < nv1);
                        const float p0 = v0 ? ex2_approx(fmaf(__uint_as_float(s[c]), kScaleLog2, -m_ref)) : 0.f;
                        const float p1 = v1 ? ex2_approx(fmaf(__uint_as_float(s[c + 1]), kScaleLog2, -m_ref)) : 0.f;
                        rs += p0 + p1;
                        s[c / 2] = pack_half2(p0, p1);
                    }
                }
            } else if (full) {
                // packed fp32 pair arithmetic: half the issue slots of scalar FMA / add
                float2 r2[4];   // independent partial sums
#pragma unroll
                for (int i = 0; i < 4; ++i) r2[i] = make_float2(0.f, 0.f);
                const float2 scale2 = make_float2(kScaleLog2, kScaleLog2);
                const float2 shift2 = make_float2(-m_ref, -m_ref);
#pragma unroll
                for (int c = 0; c < BKV; c += 2) {
                    const int i = c / 2;
                    const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                                scale2, shift2);
                    const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    r2[i & 3] = __fadd2_rn(r2[i & 3], pr);
                    s[i] = pack_half2(pr.x, pr.y);
                }
                rs = ((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y)) + ((r2[2].x + r2[2].y) + (r2[3].x + r2[3].y));
            } else {
#pragma unroll
                for (int c = 0; c < BKV; c += 2) {
                    const float p0 =
                        member && c < nvalid ? ex2_approx(fmaf(__uint_as_float(s[c]), kScaleLog2, -m_ref)) : 0.f;
                    const float p1 =
                        member && c + 1 < nvalid ? ex2_approx(fmaf(__uint_as_float(s[c + 1]), kScaleLog2, -m_ref)) : 0.f;
                    rs += p0 + p1;
                    s[c / 2] = pack_half2(p0, p1);
                }
            }
            l = l * factor + rs;
            // P.V of the previous tile must be done before O is rescaled or P overwritten
            if (u > 0 && !warp_wait(&ctl.o_done, (u - 1) & 1, abort, prm.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, corr)) {   // lazy rescale of O, before P.V of this tile
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + kColO + 32 * a, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
                    tmem_st32(lane_base + kColO + 32 * a, o);
                }
            }
#pragma unroll
            for (int c = 0; c < TC / 64; ++c)
                tmem_st32(lane_base + kColP + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&s[32 * c]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.p_full);
        }
        // ------------------------------------------------------------ epilogue
        const bool have = ok && n > 0 && warp_wait(&ctl.o_final, 0, abort, prm.status);
        if (!have) l = 0.f;   // empty row, or aborted: report an empty row
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
        if (have) tc_fence_after();
        const int qrow = tq * 128 + row;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            float o[32];
            if (have) {
                uint32_t r[32];
                tmem_ld32(lane_base + kColO + 32 * a, r);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(r[c]) * inv;
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] = 0.f;
            }
            if (MODE == MODE_SPECIAL_ALL) {
                float* dst = prm.spart + (((size_t)split * g.H + h) * pl.ns_pad + qrow) * 64 + 32 * a;
#pragma unroll
                for (int c = 0; c < 32; c += 4) Vec16<float>::store(dst + c, o + c);
            } else if (MODE == MODE_FUSED) {
                if (qrow < g.Np) {
                    __nv_bfloat16* dst = prm.out + (size_t)patch_row(g, qrow) * g.H * 64 + (size_t)h * 64 + 32 * a;
#pragma unroll
                    for (int c = 0; c < 32; c += 8) Vec16<__nv_bfloat16>::store(dst + c, o + c);
                }
            } else if (qrow < g.Np) {
                float* dst = prm.o_part + ((size_t)qrow * g.H + h) * 64 + 32 * a;
#pragma unroll
                for (int c = 0; c < 32; c += 4) Vec16<float>::store(dst + c, o + c);
            }
        }
        if (MODE == MODE_SPECIAL_ALL) prm.slse[((size_t)split * g.H + h) * pl.ns_pad + qrow] = lse;
        else if (MODE != MODE_FUSED && qrow < g.Np) prm.lse_part[(size_t)h * g.Np + qrow] = lse;
    }

    // ------------------------------------------------------------------ teardown
    __syncthreads();
    if (ctl.abort) {
        // let in-flight copies and MMAs land before the shared and tensor memory go away
        if (warp == 0 && lane == 0)
            for (int u = max(0, issued - NS); u < issued; ++u)
                drain_wait(&ctl.kv_full[u % NS], (u / NS) & 1, prm.status);
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

// Combines the key-range splits of the special queries: L = ln sum_s e^lse_s,
// out = sum_s e^(lse_s - L) O_s, written to the special rows of out (bf16).
__global__ void __launch_bounds__(256)
special_combine_kernel(Geo g, PackedLayout pl, const float* __restrict__ spart, const float* __restrict__ slse,
                       __nv_bfloat16* __restrict__ out) {
    const size_t total = (size_t)g.Ns * g.H * 8;   // (special token, head, 8-element group)
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < total;
         x += (size_t)gridDim.x * blockDim.x) {
        const int grp = (int)(x & 7);
        const size_t th = x >> 3;
        const int h = (int)(th % g.H);
        const int t = (int)(th / g.H);
        float mx = -INFINITY;
        for (int s = 0; s < pl.nsplit; ++s) mx = fmaxf(mx, slse[((size_t)s * g.H + h) * pl.ns_pad + t]);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float wsum = 0.f;
        if (mx != -INFINITY) {
            for (int s = 0; s < pl.nsplit; ++s) {
                const float w = expf(slse[((size_t)s * g.H + h) * pl.ns_pad + t] - mx);
                wsum += w;
                const float4* src =
                    reinterpret_cast<const float4*>(spart + (((size_t)s * g.H + h) * pl.ns_pad + t) * 64 + grp * 8);
                const float4 a = __ldg(src), b = __ldg(src + 1);
                acc[0] += w * a.x; acc[1] += w * a.y; acc[2] += w * a.z; acc[3] += w * a.w;
                acc[4] += w * b.x; acc[5] += w * b.y; acc[6] += w * b.z; acc[7] += w * b.w;
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= inv;
        Vec16<__nv_bfloat16>::store(out + (size_t)special_row(g, t) * g.H * 64 + (size_t)h * 64 + grp * 8, acc);
    }
}

// ---------------------------------------------------------------------- host side

template <int MODE, int BKV>
cudaError_t launch_mode(const TcParams& prm, const CUtensorMap& q, const CUtensorMap& ka, const CUtensorMap& va,
                        const CUtensorMap& kb, const CUtensorMap& vb, int ctas, cudaStream_t st) {
    if (ctas == 0) return cudaSuccess;
    const size_t smem = smem_bytes<BKV>(prm.g.B);
    auto kern = attn_tc_kernel<MODE, BKV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kThreads, smem, st>>>(q, ka, va, kb, vb, prm);
    return cudaGetLastError();
}

}  // namespace

// mode: 0 sparse (o_part/lse_part), 1 patch->special (o_part/lse_part),
//       2 special->all (out, through the split partials), 3 fused sparse + special keys (out)
cudaError_t launch_attn_tc(const Geo& g, int mode, const void* ws, const uint16_t* kv_idx,
                           const int32_t* kv_cnt, float* o_part, float* lse_part, void* out,
                           int32_t* status, cudaStream_t st) {
    const PackedLayout pl = packed_layout(g);
    uint8_t* base = static_cast<uint8_t*>(const_cast<void*>(ws));
    TcParams prm;
    prm.g = g;
    prm.pl = pl;
    prm.kv_idx = kv_idx;
    prm.kv_cnt = kv_cnt;
    prm.o_part = o_part;
    prm.lse_part = lse_part;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.spart = reinterpret_cast<float*>(base + pl.spart);
    prm.slse = reinterpret_cast<float*>(base + pl.slse);
    prm.status = status;
    const uint64_t prow = (uint64_t)g.H * pl.np_pad;
    const uint64_t srow = (uint64_t)g.H * pl.ns_pad;
    const bool has_sp = g.Ns > 0;
    CUtensorMap q, ka, va, kb, vb;
    const int patch_tiles = pl.np_pad / 128;
    if (mode == MODE_SPARSE || mode == MODE_FUSED) {
        if (!make_tile_map(&q, base + pl.qp, prow, 64, 128, false) || !make_tile_map(&kb, base + pl.kp, prow, 64, g.b, false) ||
            !make_tile_map(&vb, base + pl.vp, prow, 64, g.b, true))
            return cudaErrorInvalidValue;
        if (mode == MODE_FUSED && has_sp) {
            if (!make_tile_map(&ka, base + pl.ks, srow, 64, g.b, false) || !make_tile_map(&va, base + pl.vs, srow, 64, g.b, true))
                return cudaErrorInvalidValue;
        } else {
            ka = kb;
            va = vb;
        }
        prm.q_tiles = patch_tiles;
        const int ctas = patch_tiles * g.H;
        if (mode == MODE_SPARSE)
            return g.b == 128 ? launch_mode<MODE_SPARSE, 128>(prm, q, ka, va, kb, vb, ctas, st)
                              : launch_mode<MODE_SPARSE, 64>(prm, q, ka, va, kb, vb, ctas, st);
        return g.b == 128 ? launch_mode<MODE_FUSED, 128>(prm, q, ka, va, kb, vb, ctas, st)
                          : launch_mode<MODE_FUSED, 64>(prm, q, ka, va, kb, vb, ctas, st);
    }
    if (!has_sp) return cudaSuccess;
    if (!make_tile_map(&ka, base + pl.ks, srow, 64, 128, false) || !make_tile_map(&va, base + pl.vs, srow, 64, 128, true))
        return cudaErrorInvalidValue;
    if (mode == MODE_PATCH_SPECIAL) {
        if (!make_tile_map(&q, base + pl.qp, prow, 64, 128, false)) return cudaErrorInvalidValue;
        prm.q_tiles = patch_tiles;
        return launch_mode<MODE_PATCH_SPECIAL, 128>(prm, q, ka, va, ka, va, patch_tiles * g.H, st);
    }
    if (!make_tile_map(&q, base + pl.qs, srow, 64, 128, false) || !make_tile_map(&kb, base + pl.kp, prow, 64, 128, false) ||
        !make_tile_map(&vb, base + pl.vp, prow, 64, 128, true))
        return cudaErrorInvalidValue;
    prm.q_tiles = pl.ns_pad / 128;
    cudaError_t e = launch_mode<MODE_SPECIAL_ALL, 128>(prm, q, ka, va, kb, vb, prm.q_tiles * pl.nsplit * g.H, st);
    if (e != cudaSuccess) return e;
    special_combine_kernel<<<num_sms() * 4, 256, 0, st>>>(g, pl, prm.spart, prm.slse, prm.out);
    return cudaGetLastError();
}

}  // namespace bsa
