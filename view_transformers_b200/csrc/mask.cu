// Block-mask prediction ("Block-Sparse Global Attention for Efficient Multi-View Geometry
// Transformers", 关键设计 1 and 2): pooled scores s_ij = <PQ_hi, PK_hj> / sqrt(d), their
// row softmax p_ij, and the Top-K + CDF dual threshold: keep the first
// n = min(B, max(k_h, n_tau)) blocks of the ranking (p descending, lower index first),
// n_tau = smallest n with cumulative mass >= tau.
//
// One warp per query-block row, W rows (warps) of one head per CTA so that each PK tile
// staged in shared memory serves W rows. The [H, B, B] score matrix is never written to
// HBM. Instead of sorting a row, the selection is a radix select on the order-preserving
// 32-bit image of the fp32 score:
//   - the common leading bits of the row's keys are skipped (near-uniform rows share
//     sign and exponent), then 8-bit digits are resolved from the top;
//   - the CDF bound uses per-digit fp64 mass histograms (the target is tau * sum_j e_j,
//     e_j = exp(s_ij - max_j s_ij), so no division is needed);
//   - ties (equal keys) are taken in ascending block index.
// The kept blocks are then emitted in ascending index order with warp ballots.
#include <cfloat>

#include "common.cuh"

namespace bsa {
namespace {

constexpr int kKeyTile = 64;      // PK rows staged per pass
constexpr int kPkStride = 68;     // padded row (floats): conflict-free 16-byte loads
constexpr int kRadix = 256;

struct WarpHist {
    unsigned int cnt[kRadix];
    double mass[kRadix];
};

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Result of a descending radix select over a row's keys.
struct Cut {
    uint32_t t;        // threshold key
    int greater;       // elements with key > t
    int take;          // elements with key == t that are kept (lowest indices first)
};

// Finds the cut for either the n largest keys (mass_mode = false, target_n) or the smallest
// prefix of the ranking whose mass reaches target_m (mass_mode = true). Warp-collective.
__device__ Cut radix_cut(const uint32_t* keys, const float* e, int B, bool mass_mode, int target_n,
                         double target_m, WarpHist* hist, int lane) {
    // common prefix of all keys
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = lane; j < B; j += 32) {
        kmin = min(kmin, keys[j]);
        kmax = max(kmax, keys[j]);
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
    int greater = 0;
    int rem_n = target_n;
    double rem_m = target_m;

    while (hb >= 0) {
        if (mass_mode && rem_m <= 0.0) {   // rounding left no mass to cover: keep one more
            mass_mode = false;
            rem_n = 1;
        }
        const int width = hb + 1 >= 8 ? 8 : hb + 1;
        const int shift = hb + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int x = lane; x < kRadix; x += 32) {
            hist->cnt[x] = 0u;
            hist->mass[x] = 0.0;
        }
        __syncwarp();
        for (int j = lane; j < B; j += 32) {
            const uint32_t u = keys[j];
            if ((u & fixed_mask) == prefix) {
                const int dg = (u >> shift) & dmask;
                atomicAdd(&hist->cnt[dg], 1u);
                if (mass_mode) atomicAdd(&hist->mass[dg], (double)e[j]);
            }
        }
        __syncwarp();
        // lane l owns digits 255-8l .. 248-8l (descending); exclusive scan in lane order
        unsigned c[8];
        double m[8];
        unsigned lc = 0;
        double lm = 0.0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int dg = kRadix - 1 - (8 * lane + q);
            c[q] = hist->cnt[dg];
            m[q] = mass_mode ? hist->mass[dg] : 0.0;
            lc += c[q];
            lm += m[q];
        }
        unsigned ic = lc;
        double im = lm;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned oc = __shfl_up_sync(0xffffffffu, ic, o);
            const double om = __shfl_up_sync(0xffffffffu, im, o);
            if (lane >= o) { ic += oc; im += om; }
        }
        unsigned ec = __shfl_up_sync(0xffffffffu, ic, 1);
        double em = __shfl_up_sync(0xffffffffu, im, 1);
        if (lane == 0) { ec = 0u; em = 0.0; }
        const bool hit = lc > 0 && (mass_mode ? (em < rem_m && rem_m <= im)
                                              : (ec < (unsigned)rem_n && (unsigned)rem_n <= ic));
        const unsigned hits = __ballot_sync(0xffffffffu, hit);
        // no lane reaches the target (mass above the histogram total by rounding): cut at
        // the lowest non-empty digit, which keeps every candidate.
        const int src = hits ? __ffs(hits) - 1 : 31 - __clz(__ballot_sync(0xffffffffu, lc > 0));
        int dsel = 0;
        unsigned above_c = 0;
        double above_m = 0.0;
        if (lane == src) {
            int qsel = -1;
            if (hits) {
                unsigned accc = ec;
                double accm = em;
                for (int q = 0; q < 8 && qsel < 0; ++q) {
                    if (mass_mode ? (accm + m[q] >= rem_m) : (accc + c[q] >= (unsigned)rem_n)) qsel = q;
                    else { accc += c[q]; accm += m[q]; }
                }
            }
            if (qsel < 0)
                for (int q = 0; q < 8; ++q) if (c[q] > 0) qsel = q;   // lowest non-empty digit
            above_c = ec;
            above_m = em;
            for (int q = 0; q < qsel; ++q) { above_c += c[q]; above_m += m[q]; }
            dsel = kRadix - 1 - (8 * lane + qsel);
        }
        dsel = __shfl_sync(0xffffffffu, dsel, src);
        above_c = __shfl_sync(0xffffffffu, above_c, src);
        above_m = __shfl_sync(0xffffffffu, above_m, src);
        greater += (int)above_c;
        rem_n -= (int)above_c;
        rem_m -= above_m;
        prefix |= ((uint32_t)dsel) << shift;
        fixed_mask |= dmask << shift;
        hb = shift - 1;
        __syncwarp();
    }
    // every key equal to `prefix` is now a tie at the cut
    int ties = 0;
    float et = 0.f;
    for (int j = lane; j < B; j += 32) {
        if (keys[j] == prefix) { ++ties; et = e[j]; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ties += __shfl_xor_sync(0xffffffffu, ties, o);
        et = fmaxf(et, __shfl_xor_sync(0xffffffffu, et, o));
    }
    Cut cut;
    cut.t = prefix;
    cut.greater = greater;
    if (mass_mode) {
        int need = rem_m <= 0.0 ? 1 : (int)ceil(rem_m / (double)et);
        cut.take = max(1, min(ties, need));
    } else {
        cut.take = max(0, min(ties, rem_n));
    }
    return cut;
}

__global__ void mask_kernel(Geo g, MaskParams mp, const float* __restrict__ pq,
                            const float* __restrict__ pk, uint32_t* __restrict__ mask_bits,
                            uint16_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
                            int32_t* status) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int W = blockDim.x / 32;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int h = blockIdx.y;
    const int B = g.B;
    const int i = blockIdx.x * W + warp;           // query block of this warp
    const bool row_ok = i < B;

    float* pk_tile = reinterpret_cast<float*>(smem);                    // [kKeyTile][kPkStride]
    float* pq_rows = pk_tile + kKeyTile * kPkStride;                      // [W][64]
    WarpHist* hists = reinterpret_cast<WarpHist*>(pq_rows + W * 64);      // [W]
    unsigned char* rowbuf = reinterpret_cast<unsigned char*>(hists + W);  // [W][B] keys, [W][B] e
    uint32_t* keys = reinterpret_cast<uint32_t*>(rowbuf) + (size_t)warp * B;
    float* ex = reinterpret_cast<float*>(rowbuf + (size_t)W * B * 4) + (size_t)warp * B;
    float* sc = ex;   // scores are kept in the e buffer until the softmax pass

    const float* pk_h = pk + (size_t)h * B * 64;
    for (int x = lane; x < 64; x += 32) pq_rows[warp * 64 + x] = row_ok ? pq[((size_t)h * B + i) * 64 + x] : 0.f;
    const float scale = 0.125f;   // 1 / sqrt(64)

    // ---- pooled scores, one 64-row PK tile at a time
    for (int j0 = 0; j0 < B; j0 += kKeyTile) {
        __syncthreads();
        const int nrows = min(kKeyTile, B - j0);
        for (int x = threadIdx.x; x < nrows * 16; x += blockDim.x) {
            const int r = x / 16, c4 = x % 16;
            const float4 v = __ldg(reinterpret_cast<const float4*>(pk_h + (size_t)(j0 + r) * 64) + c4);
            *reinterpret_cast<float4*>(pk_tile + r * kPkStride + c4 * 4) = v;
        }
        __syncthreads();
        if (row_ok) {
            const float4* qv = reinterpret_cast<const float4*>(pq_rows + warp * 64);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = lane + 32 * half;
                if (r < nrows) {
                    const float4* kv = reinterpret_cast<const float4*>(pk_tile + r * kPkStride);
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        const float4 qa = qv[c4];
                        const float4 ka = kv[c4];
                        a0 = fmaf(qa.x, ka.x, a0);
                        a1 = fmaf(qa.y, ka.y, a1);
                        a2 = fmaf(qa.z, ka.z, a2);
                        a3 = fmaf(qa.w, ka.w, a3);
                    }
                    sc[j0 + r] = ((a0 + a1) + (a2 + a3)) * scale;
                }
            }
        }
    }
    if (!row_ok) return;
    __syncwarp();

    // ---- softmax pieces: row max, e_j = exp(s_j - max), fp64 total
    float mx = -FLT_MAX;
    for (int j = lane; j < B; j += 32) mx = fmaxf(mx, sc[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double tot = 0.0;
    for (int j = lane; j < B; j += 32) {
        const float s = sc[j];
        keys[j] = order_key(s);
        const float e = expf(s - mx);
        ex[j] = e;
        tot += (double)e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    __syncwarp();

    // ---- dual threshold
    const int k = mp.k[h];
    WarpHist* hist = hists + warp;
    int n;
    Cut cut;
    bool have_cut = false;
    if (mp.tau > 0.0) {
        cut = radix_cut(keys, ex, B, true, 0, mp.tau * tot, hist, lane);
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
            cut = radix_cut(keys, ex, B, false, n, 0.0, hist, lane);
        }
    }
    const bool none = n <= 0;

    // ---- emit: ascending indices, bit mask, count
    const int words = (B + 31) / 32;
    uint16_t* out_idx = kv_idx + ((size_t)h * B + i) * B;
    int taken_ties = 0, written = 0;
    for (int j0 = 0; j0 < B; j0 += 32) {
        const int j = j0 + lane;
        const bool valid = j < B;
        const uint32_t u = valid ? keys[j] : 0u;
        const bool tie = valid && !none && u == cut.t;
        const unsigned tb = __ballot_sync(0xffffffffu, tie);
        const int trank = taken_ties + __popc(tb & lanemask_lt());
        taken_ties += __popc(tb);
        const bool sel = valid && !none && (u > cut.t || (tie && trank < cut.take));
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

}  // namespace

cudaError_t launch_mask(const Geo& g, const MaskParams& mp, const float* pq, const float* pk,
                        uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                        int32_t* status, cudaStream_t st) {
    const size_t fixed = (size_t)kKeyTile * kPkStride * 4;
    const size_t per_warp = 64 * 4 + sizeof(WarpHist) + (size_t)g.B * 8;
    const size_t budget = 200 * 1024;
    int W = (int)((budget - fixed) / per_warp);
    W = W > 8 ? 8 : W;
    if (W < 1) return cudaErrorInvalidValue;
    const size_t smem = fixed + W * per_warp;
    cudaError_t e = cudaFuncSetAttribute(mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((g.B + W - 1) / W, g.H);
    mask_kernel<<<grid, 32 * W, smem, st>>>(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status);
    return cudaGetLastError();
}

}  // namespace bsa
