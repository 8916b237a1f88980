// Block-mask prediction ("Block-Sparse Global Attention for Efficient Multi-View Geometry
// Transformers", 关键设计 1 and 2): pooled scores s_ij = <PQ_hi, PK_hj> / sqrt(d), their
// row softmax p_ij, and the Top-K + CDF dual threshold: keep the first
// n = min(B, max(k_h, n_tau)) blocks of the ranking (p descending, lower index first),
// n_tau = smallest n with cumulative mass >= tau.
//
// One CTA holds R query-block rows of one head. The [H, B, B] score matrix is never
// written to HBM: a CTA computes its R x B score rows into shared memory, then each warp
// selects on one row at a time.
//
// Scores (FMA-bound): pooled K is stored dimension-major ([H][d][B]), so a warp reads 32
// consecutive blocks of one dimension per load straight from L2; each lane accumulates
// one block x 8 rows (8 independent FMA chains) with the query values of a dimension
// broadcast from shared memory (one shared-memory wavefront feeds 4 FMAs per lane). The
// kernel stays within 64 registers and about 46 KB of shared memory at B = 608, so four
// 8-warp CTAs share an SM and cover each other's barrier between the two phases.
//
// Selection: instead of sorting a row, a select over the fp32 scores in three steps:
//   - one pass counts the row into 256 equal-width score buckets over [min, max] (with
//     tau > 0 also their masses e_j = exp(s_ij - max_j s_ij)); the bucket where the
//     running count reaches k, or the running mass reaches tau * sum_j e_j, holds the cut
//     (the CDF bound needs no division);
//   - a bucket of at most 32 members is finished by ranking its members against each other
//     in one warp; a larger one by a radix select on the order-preserving 32-bit image of
//     the scores of its members (common leading bits skipped, then 8-bit digits);
//   - ties (equal scores) are taken in ascending block index.
// Masses are summed as fixed-point integers, so every sum is exact and independent of the
// order in which shared-memory atomics land. The kept blocks are then emitted in ascending
// index order with warp ballots.
#include <cfloat>

#include "common.cuh"

namespace bsa {
namespace {

constexpr int kWarps = 8;         // per CTA; one query-block row each
constexpr int kRadix = 256;
constexpr int kDim = 64;

// Masses are fixed-point: e_j * 2^40 rounded to an integer. With at most 2^13 blocks every
// partial sum is an integer below 2^53, so the sums are exact in any order (atomics stay
// deterministic) and convert to double without rounding.
constexpr float kFix = 1099511627776.0f;   // 2^40

struct WarpHist {
    unsigned int cnt[kRadix];
    unsigned long long mass[kRadix];
};

// Order-preserving 32-bit image of a score; -0 and +0 (equal scores) map to one key.
__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

__device__ __forceinline__ unsigned long long fix_mass(float s, float mx) {
    return __float2ull_rn(expf(s - mx) * kFix);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Equal-width score buckets over [lo, max]: digit(s) = min(255, floor((s - lo) * scale)) is
// monotone in s, so a higher bucket holds strictly larger scores and equal scores share a
// bucket. sel >= 0 restricts a pass to the members of one bucket.
struct Bucket {
    float lo, scale;
    int sel;
    __device__ __forceinline__ int digit(float s) const {
        return min(kRadix - 1, __float2int_rz((s - lo) * scale));
    }
    __device__ __forceinline__ bool member(float s) const { return sel < 0 || digit(s) == sel; }
};

// Result of a descending selection over a row.
struct Cut {
    uint32_t t;        // threshold key
    int greater;       // elements with key > t
    int take;          // elements with key == t that are kept (lowest indices first)
};

// One digit of a descending select: the digit where the running count reaches rem_n
// (mass_mode = false) or the running mass reaches rem_m, with what lies above it.
struct Pick {
    int digit;
    unsigned above_c, at_c;
    double above_m;
};

__device__ Pick scan_hist(const WarpHist* hist, bool mass_mode, int rem_n, double rem_m, int lane) {
    // lane l owns digits 255-8l .. 248-8l (descending); exclusive scan in lane order
    unsigned c[8];
    double m[8];
    unsigned lc = 0;
    double lm = 0.0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int dg = kRadix - 1 - (8 * lane + q);
        c[q] = hist->cnt[dg];
        m[q] = mass_mode ? (double)hist->mass[dg] : 0.0;
        lc += c[q];
        lm += m[q];
    }
    unsigned ic = lc;
    double im = lm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned oc = __shfl_up_sync(0xffffffffu, ic, o);
        const double om = mass_mode ? __shfl_up_sync(0xffffffffu, im, o) : 0.0;
        if (lane >= o) { ic += oc; im += om; }
    }
    const unsigned ec = ic - lc;
    const double em = im - lm;     // exact: integers below 2^53
    const bool hit = lc > 0 && (mass_mode ? (em < rem_m && rem_m <= im)
                                          : (ec < (unsigned)rem_n && (unsigned)rem_n <= ic));
    const unsigned hits = __ballot_sync(0xffffffffu, hit);
    // no lane reaches the target: cut at the lowest non-empty digit (keeps every candidate)
    const int src = hits ? __ffs(hits) - 1 : 31 - __clz(__ballot_sync(0xffffffffu, lc > 0));
    Pick pk{0, 0u, 0u, 0.0};
    if (lane == src) {
        unsigned accc = ec;
        double accm = em;
        int qsel = -1;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const bool here = hits ? (qsel < 0 && (mass_mode ? (accm + m[q] >= rem_m)
                                                            : (accc + c[q] >= (unsigned)rem_n)))
                                   : c[q] > 0;   // fallback: the last non-empty digit wins
            if (here) {
                qsel = q;
                pk.above_c = accc;
                pk.above_m = accm;
                pk.at_c = c[q];
            }
            if (qsel < 0 || !hits) { accc += c[q]; accm += m[q]; }
        }
        pk.digit = kRadix - 1 - (8 * lane + qsel);
    }
    pk.digit = __shfl_sync(0xffffffffu, pk.digit, src);
    pk.above_c = __shfl_sync(0xffffffffu, pk.above_c, src);
    pk.at_c = __shfl_sync(0xffffffffu, pk.at_c, src);
    if (mass_mode) pk.above_m = __shfl_sync(0xffffffffu, pk.above_m, src);
    return pk;
}

// Radix select over the order-preserving keys of the candidates (members of f, ncand of
// them), below `greater` elements already kept: the cut for rem_n more elements
// (mass_mode = false) or for rem_m more mass. Warp-collective.
__device__ Cut radix_cut(const float* s, int B, float mx, Bucket f, int ncand, bool mass_mode,
                         int greater, int rem_n, double rem_m, WarpHist* hist, int lane) {
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = lane; j < B; j += 32) {
        const float sj = s[j];
        if (f.member(sj)) {
            const uint32_t u = order_key(sj);
            kmin = min(kmin, u);
            kmax = max(kmax, u);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    const uint32_t diff = kmin ^ kmax;
    int hb = diff ? 31 - __clz(diff) : -1;      // highest differing bit
    uint32_t fixed_mask = hb >= 31 ? 0u : (0xffffffffu << (hb + 1));
    uint32_t prefix = kmax & fixed_mask;
    int ties = ncand;                            // all candidates equal when no digit is resolved

    while (hb >= 0) {
        if (mass_mode && rem_m <= 0.0) {   // nothing left to cover: keep one more
            mass_mode = false;
            rem_n = 1;
        }
        const int width = hb + 1 >= 8 ? 8 : hb + 1;
        const int shift = hb + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        __syncwarp();
        for (int x = lane; x < kRadix; x += 32) {
            hist->cnt[x] = 0u;
            if (mass_mode) hist->mass[x] = 0ull;
        }
        __syncwarp();
        for (int j = lane; j < B; j += 32) {
            const float sj = s[j];
            const uint32_t u = order_key(sj);
            if ((u & fixed_mask) == prefix && f.member(sj)) {
                const int dg = (u >> shift) & dmask;
                atomicAdd(&hist->cnt[dg], 1u);
                if (mass_mode) atomicAdd(&hist->mass[dg], fix_mass(sj, mx));
            }
        }
        __syncwarp();
        const Pick pk = scan_hist(hist, mass_mode, rem_n, rem_m, lane);
        greater += (int)pk.above_c;
        rem_n -= (int)pk.above_c;
        rem_m -= pk.above_m;
        prefix |= ((uint32_t)pk.digit) << shift;
        fixed_mask |= dmask << shift;
        ties = (int)pk.at_c;        // after the last digit: the candidates equal to prefix
        hb = shift - 1;
    }
    Cut cut;
    cut.t = prefix;
    cut.greater = greater;
    if (mass_mode) {
        const double et = (double)fix_mass(key_value(prefix), mx);
        const int need = rem_m <= 0.0 ? 1 : et > 0.0 ? (int)ceil(rem_m / et) : ties;
        cut.take = max(1, min(ties, need));
    } else {
        cut.take = max(0, min(ties, rem_n));
    }
    return cut;
}

// The cut inside one bucket of at most 32 members: each lane takes one member and ranks it
// against the others (score descending, index ascending).
__device__ Cut small_cut(const float* s, int B, float mx, Bucket f, int m, bool mass_mode,
                         int greater, int rem_n, double rem_m, WarpHist* hist, int lane) {
    float* ls = reinterpret_cast<float*>(hist->cnt);      // [32] member scores
    int* lj = reinterpret_cast<int*>(hist->cnt) + 32;     // [32] member indices
    __syncwarp();
    int base = 0;
    for (int j0 = 0; j0 < B; j0 += 32) {
        const int j = j0 + lane;
        const float sj = j < B ? s[j] : 0.f;
        const bool pred = j < B && f.digit(sj) == f.sel;
        const unsigned bal = __ballot_sync(0xffffffffu, pred);
        const int pos = base + __popc(bal & lanemask_lt());
        if (pred && pos < 32) { ls[pos] = sj; lj[pos] = j; }
        base += __popc(bal);
    }
    __syncwarp();
    const bool mine = lane < m;
    const float cs = mine ? ls[lane] : -FLT_MAX;
    const int cj = mine ? lj[lane] : 0x7fffffff;
    const unsigned long long ce = (mass_mode && mine) ? fix_mass(cs, mx) : 0ull;
    int rank = 0;
    unsigned long long before = 0ull;
    for (int t = 0; t < m; ++t) {
        const float st = __shfl_sync(0xffffffffu, cs, t);
        const int jt = __shfl_sync(0xffffffffu, cj, t);
        const unsigned long long et = mass_mode ? __shfl_sync(0xffffffffu, ce, t) : 0ull;
        if (st > cs || (st == cs && jt < cj)) { ++rank; before += et; }
    }
    const bool sel = mine && (mass_mode ? (double)before < rem_m : rank < rem_n);
    const int nsel = __popc(__ballot_sync(0xffffffffu, sel));
    // the last kept member (rank nsel - 1), or the first member when none is kept
    const unsigned lastb = __ballot_sync(0xffffffffu, mine && rank == (nsel > 0 ? nsel - 1 : 0));
    const uint32_t kt = order_key(__shfl_sync(0xffffffffu, cs, __ffs(lastb) - 1));
    const int take = __popc(__ballot_sync(0xffffffffu, sel && order_key(cs) == kt));
    Cut cut;
    cut.t = kt;
    cut.greater = greater + nsel - take;
    cut.take = take;
    return cut;
}

// Selection and emission for one row (h, i) whose scores are s[0, B).
__device__ void select_row(const float* s, int B, int h, int i, int k, double tau,
                           WarpHist* hist, uint32_t* __restrict__ mask_bits,
                           uint16_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
                           int32_t* status, int lane) {
    float fmin = FLT_MAX, fmax = -FLT_MAX;
    for (int j = lane; j < B; j += 32) {
        const float sj = s[j];
        fmin = fminf(fmin, sj);
        fmax = fmaxf(fmax, sj);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        fmin = fminf(fmin, __shfl_xor_sync(0xffffffffu, fmin, o));
        fmax = fmaxf(fmax, __shfl_xor_sync(0xffffffffu, fmax, o));
    }
    const uint32_t kmin = order_key(fmin), kmax = order_key(fmax);
    const float mx = key_value(kmax);
    const float smin = key_value(kmin);
    const float scale = (float)kRadix / (mx - smin);
    // equal-width buckets unless the range is zero (all equal, or only +0 / -0) or too
    // narrow for a finite scale; the radix select then works on the key bits directly
    const bool bucketed = kmin != kmax && isfinite(scale);
    const Bucket all{smin, scale, -1};

    // The cut for the first n_target elements (mass_mode = false) or for mass tau * T,
    // T = sum_j e_j (mass_mode = true).
    auto find_cut = [&](bool mass_mode, int n_target) -> Cut {
        if (!bucketed) {
            double rem_m = 0.0;
            if (mass_mode) {
                unsigned long long tot = 0ull;
                for (int j = lane; j < B; j += 32) tot += fix_mass(s[j], mx);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
                rem_m = tau * (double)tot;
            }
            return radix_cut(s, B, mx, all, B, mass_mode, 0, n_target, rem_m, hist, lane);
        }
        __syncwarp();
        for (int x = lane; x < kRadix; x += 32) {
            hist->cnt[x] = 0u;
            if (mass_mode) hist->mass[x] = 0ull;
        }
        __syncwarp();
        for (int j = lane; j < B; j += 32) {
            const float sj = s[j];
            const int dg = all.digit(sj);
            atomicAdd(&hist->cnt[dg], 1u);
            if (mass_mode) atomicAdd(&hist->mass[dg], fix_mass(sj, mx));
        }
        __syncwarp();
        double rem_m = 0.0;
        if (mass_mode) {
            unsigned long long tot = 0ull;
            for (int x = lane; x < kRadix; x += 32) tot += hist->mass[x];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
            rem_m = tau * (double)tot;
        }
        const Pick pk = scan_hist(hist, mass_mode, n_target, rem_m, lane);
        const Bucket f{smin, scale, pk.digit};
        const int greater = (int)pk.above_c;
        const int rem_n = n_target - (int)pk.above_c;
        rem_m -= pk.above_m;
        if (pk.at_c <= 32)
            return small_cut(s, B, mx, f, (int)pk.at_c, mass_mode, greater, rem_n, rem_m, hist, lane);
        return radix_cut(s, B, mx, f, (int)pk.at_c, mass_mode, greater, rem_n, rem_m, hist, lane);
    };

    int n;
    Cut cut;
    bool have_cut = false;
    if (tau > 0.0) {
        cut = find_cut(true, 0);
        const int n_tau = cut.greater + cut.take;
        if (n_tau >= k) {
            n = n_tau;
            have_cut = true;
        } else {
            n = k;
        }
    } else {
        n = k;
    }
    n = min(n, B);
    if (!have_cut) {
        if (n <= 0) {
            cut.t = 0xffffffffu; cut.greater = 0; cut.take = 0;    // nothing above or at the cut
        } else {
            cut = find_cut(false, n);
        }
    }
    const bool none = n <= 0;

    // ---- emit: ascending indices, bit mask, count
    const int words = (B + 31) / 32;
    uint16_t* out_idx = kv_idx + ((size_t)h * B + i) * B;
    int taken_ties = 0, written = 0;
    const float tval = key_value(cut.t);   // score comparisons agree with key comparisons
    for (int j0 = 0; j0 < B; j0 += 32) {
        const int j = j0 + lane;
        const bool valid = j < B && !none;
        const float sj = valid ? s[j] : 0.f;
        const bool tie = valid && sj == tval;
        const unsigned tb = __ballot_sync(0xffffffffu, tie);
        const int trank = taken_ties + __popc(tb & lanemask_lt());
        taken_ties += __popc(tb);
        const bool sel = valid && (sj > tval || (tie && trank < cut.take));
        const unsigned sb = __ballot_sync(0xffffffffu, sel);
        if (sel) out_idx[written + __popc(sb & lanemask_lt())] = (uint16_t)j;
        written += __popc(sb);
        if (mask_bits != nullptr && lane == 0) mask_bits[((size_t)h * B + i) * words + j0 / 32] = sb;
    }
    if (lane == 0) {
        kv_cnt[(size_t)h * B + i] = written;
        if (written != n) record_error(status, BSA_ERR_DEVICE_BOUNDS);
    }
}

// Row stride of the transposed query block in shared memory: 16-byte aligned rows.
template <int R>
__host__ __device__ constexpr int q_stride() { return (R + 3) / 4 * 4; }

// R query-block rows i0 .. i0+R-1 of head h per CTA, on W warps (at most 16; MINB CTAs per
// SM in the launch bounds).
template <int R, int W, int MINB>
__global__ void __launch_bounds__(32 * W, MINB)
mask_kernel(Geo g, MaskParams mp, const float* __restrict__ pq, const float* __restrict__ pk,
            uint32_t* __restrict__ mask_bits, uint16_t* __restrict__ kv_idx,
            int32_t* __restrict__ kv_cnt, int32_t* status) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int h = blockIdx.y;
    const int B = g.B;
    const int i0 = blockIdx.x * R;

    constexpr int QS = q_stride<R>();
    float* qT = reinterpret_cast<float*>(smem);                        // [d][QS]
    WarpHist* hists = reinterpret_cast<WarpHist*>(qT + kDim * QS);     // [W]
    float* sc = reinterpret_cast<float*>(hists + W);                   // [R][B]

    for (int x = threadIdx.x; x < R * kDim; x += blockDim.x) {
        const int r = x / kDim, d = x % kDim;
        qT[d * QS + r] = i0 + r < B ? pq[((size_t)h * B + i0 + r) * kDim + d] : 0.f;
    }
    __syncthreads();

    // ---- pooled scores: work items of 32 blocks (one per lane) x RG rows, round-robin over
    // the warps (consecutive warps take consecutive block chunks)
    // rows per work item (R is a multiple of RG): every row at once, unless several CTAs
    // share the SM and registers cap the accumulators at 9
    constexpr int RG = (MINB == 1 || R <= 9) ? R : 8;
    const float* pk_h = pk + (size_t)h * kDim * B;
    const float scale = 0.125f;   // 1 / sqrt(64)
    const int nchunk = (B + 31) / 32;
    const int items = nchunk * (R / RG);
    for (int it = warp; it < items; it += W) {
        const int c = it % nchunk;
        const int rg = it / nchunk;
        const int j = c * 32 + lane;
        const bool valid = j < B;
        const float* p = pk_h + (valid ? j : 0);
        float a[RG];
#pragma unroll
        for (int r = 0; r < RG; ++r) a[r] = 0.f;
        float kc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) kc[u] = __ldg(p + (size_t)u * B);
#pragma unroll 1
        for (int d0 = 0; d0 < kDim; d0 += 8) {
            float kn[8];
            if (d0 + 8 < kDim) {   // next eight dimensions in flight during this group's FMAs
#pragma unroll
                for (int u = 0; u < 8; ++u) kn[u] = __ldg(p + (size_t)(d0 + 8 + u) * B);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float* qd = qT + (d0 + u) * QS + rg * RG;
#pragma unroll
                for (int r4 = 0; r4 < RG; r4 += 4) {
                    constexpr int kAll4 = RG >= 4;
                    float qv[4];
                    if (kAll4 && r4 + 4 <= RG) {   // 16-byte aligned: QS and RG (1, 2, 4, 8) keep it
                        const float4 t = *reinterpret_cast<const float4*>(qd + r4);
                        qv[0] = t.x; qv[1] = t.y; qv[2] = t.z; qv[3] = t.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) qv[e] = r4 + e < RG ? qd[r4 + e] : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (r4 + e < RG) a[r4 + e] = fmaf(qv[e], kc[u], a[r4 + e]);
                }
            }
            if (d0 + 8 < kDim) {
#pragma unroll
                for (int u = 0; u < 8; ++u) kc[u] = kn[u];
            }
        }
        if (valid) {
#pragma unroll
            for (int r = 0; r < RG; ++r) sc[(size_t)(rg * RG + r) * B + j] = a[r] * scale;
        }
    }
    __syncthreads();

    // ---- selection: warp w takes rows w, w + W, ...
    for (int r = warp; r < R; r += W) {
        const int i = i0 + r;
        if (i >= B) break;
        select_row(sc + (size_t)r * B, B, h, i, mp.k[h], mp.tau, hists + warp, mask_bits, kv_idx,
                   kv_cnt, status, lane);
    }
}

template <int R>
size_t mask_smem(int B, int W) {
    return (size_t)kDim * q_stride<R>() * 4 + sizeof(WarpHist) * W + (size_t)R * B * 4;
}

template <int R, int W, int MINB>
cudaError_t launch_rows(const Geo& g, const MaskParams& mp, const float* pq, const float* pk,
                        uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt, int32_t* status,
                        cudaStream_t st) {
    const size_t smem = mask_smem<R>(g.B, W);
    auto kern = mask_kernel<R, W, MINB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((g.B + R - 1) / R, g.H);
    kern<<<grid, 32 * W, smem, st>>>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mask(const Geo& g, const MaskParams& mp, const float* pq, const float* pk,
                        uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                        int32_t* status, cudaStream_t st) {
    // 8 rows on 8 warps: one row per warp in the selection (a chain of dependent warp-wide
    // steps), and small CTAs so that four share an SM (64 registers per thread) and cover
    // each other's barrier. When the rows leave a small last round of CTAs (e.g. 2.05 rounds
    // of 4 x 148 CTAs at 100 frames), 9 rows on 9 warps (at most 56 registers, so that four
    // CTAs still fit) finish in one round fewer.
    // With long rows only one CTA fits on an SM: as many rows as fit (one warp each).
    const size_t per_sm = 228 * 1024;
    const int slots = num_sms() * 4;
    const long long ctas8 = (long long)((g.B + 7) / 8) * g.H, ctas9 = (long long)((g.B + 8) / 9) * g.H;
    if (4 * (mask_smem<9>(g.B, 9) + 1024) <= per_sm && (ctas9 + slots - 1) / slots < (ctas8 + slots - 1) / slots)
        return launch_rows<9, 9, 4>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    const bool small = mask_smem<8>(g.B, kWarps) <= 113 * 1024;
    // the most rows per CTA whose score rows fit in shared memory
    const size_t limit = 227 * 1024;
    // (the launch bounds keep every variant within 64 registers per thread)
    if (small) return launch_rows<8, kWarps, 4>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    // Long rows: one CTA per SM, one warp per row in both phases (no warp idles during the
    // selection), all rows of the CTA in each score work item (one pass over pooled K)
    if (mask_smem<14>(g.B, 14) <= limit)
        return launch_rows<14, 14, 1>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    if (mask_smem<12>(g.B, 12) <= limit)
        return launch_rows<12, 12, 1>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    if (mask_smem<8>(g.B, 2 * kWarps) <= limit)
        return launch_rows<8, 2 * kWarps, 2>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    if (mask_smem<4>(g.B, 2 * kWarps) <= limit)
        return launch_rows<4, 2 * kWarps, 2>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    if (mask_smem<1>(g.B, 2 * kWarps) <= limit)
        return launch_rows<1, 2 * kWarps, 2>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status, st);
    return cudaErrorInvalidValue;
}

}  // namespace bsa
