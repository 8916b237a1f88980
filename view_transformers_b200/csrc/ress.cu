// Drift-score block selection ("ReSS: Residual-Restoring Sparse Attention for 3D Vision
// Transformers", 摘要, 技术框架, 关键设计): blocks are chosen by how far dropping them moves the
// attention output, with restoration rounds that refine the whole drop set. Read at the pooled
// resolution of the block-mask predictor of "Block-Sparse Global Attention for Efficient
// Multi-View Geometry Transformers" (关键设计 1). Per head h and query block i:
//   p_j     = softmax_j(PQ_i . PK_j / sqrt(d))                    (pooled probabilities)
//   o       = sum_j p_j PV_j,   delta_j = p_j (o - PV_j)          (drift vectors)
//   drift(D) = |sum_{j in D} delta_j| / (1 - sum_{j in D} p_j)    (output shift when D is dropped)
// Start by keeping the k_h blocks of largest |delta_j| (ties to the lower index); then up to
// `rounds` times restore the dropped block l giving the smallest drift and drop the kept block
// m (m != l) giving the smallest drift, keeping the swap only if the drift went down.
//
// Every decision is taken in fp64 (the pooled inputs are fp32 values, exact in fp64), so it
// agrees with an fp64 evaluation except at rounding-level ties. One CTA holds a chunk of the
// query-block rows of one head, with P_b(V) of the head staged dimension-major in shared
// memory as fp32 ([d][B]: lane j reads column j, conflict-free); one warp per row, each lane
// owning the blocks j = lane + 32 t. R . P_b(V)_j is kept for every block and updated per round
// from two rows of the fp64 Gram matrix of P_b(V) (computed first, into the workspace), so a
// round costs O(B); warp-wide argmins pick l and m.
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "select.cuh"

namespace bsa {
namespace {

constexpr int kDim = 64;

struct RessParams {
    int k[BSA_MAX_HEADS];
    int rounds;
    int rows_per_cta;
};

struct ArgMin {
    double v;
    int j;
};

__device__ __forceinline__ bool better(double v, int j, double bv, int bj) {
    return v < bv || (v == bv && j < bj);
}

// Warp-wide argmin of (value, index), ties to the lower index; every lane gets the result.
__device__ __forceinline__ ArgMin warp_argmin(double v, int j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oj = __shfl_xor_sync(0xffffffffu, j, o);
        if (better(ov, oj, v, j)) { v = ov; j = oj; }
    }
    return {v, j};
}

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ double warp_max(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmax(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Row stride of the staged P_b(V) in shared memory: odd, so that lanes reading one column of
// consecutive dimensions hit distinct banks (lanes reading consecutive blocks always do).
__host__ __device__ __forceinline__ int pv_stride(int B) { return B | 1; }

// sum_e a[e] PV[e][j] over the 64 dimensions (a in shared memory, fp64): all 64 loads issued
// first, then four independent FMA chains.
__device__ __forceinline__ double dot_col(const double* a, const float* pvt, int Bp, int j) {
    float v[kDim];
#pragma unroll
    for (int e = 0; e < kDim; ++e) v[e] = pvt[e * Bp + j];
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
    for (int e = 0; e < kDim; e += 4) {
        s0 = fma(a[e], (double)v[e], s0);
        s1 = fma(a[e + 1], (double)v[e + 1], s1);
        s2 = fma(a[e + 2], (double)v[e + 2], s2);
        s3 = fma(a[e + 3], (double)v[e + 3], s3);
    }
    return (s0 + s1) + (s2 + s3);
}

// Gram matrix of the pooled values of every head, G[h][j][m] = P_b(V)_j . P_b(V)_m in fp64
// (symmetric; row m written with consecutive j, so stores are coalesced). A round of the
// restoration then updates R . P_b(V)_j for every block from two rows of G instead of B dot
// products of length 64.
__global__ void __launch_bounds__(256)
gram_kernel(int B, const float* __restrict__ pv, double* __restrict__ G) {
    __shared__ float tj[kDim][32], tm[kDim][32];
    const int h = blockIdx.z, j0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
    const float* pvh = pv + (size_t)h * kDim * B;
    for (int x = threadIdx.x; x < kDim * 32; x += 256) {
        const int e = x / 32, c = x % 32;
        tj[e][c] = j0 + c < B ? pvh[(size_t)e * B + j0 + c] : 0.f;
        tm[e][c] = m0 + c < B ? pvh[(size_t)e * B + m0 + c] : 0.f;
    }
    __syncthreads();
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int e = 0; e < kDim; ++e) {
        const double a = tj[e][tx];
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[r] = fma(a, (double)tm[e][ty + 8 * r], acc[r]);
    }
    const int j = j0 + tx;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int m = m0 + ty + 8 * r;
        if (j < B && m < B) G[((size_t)h * B + m) * B + j] = acc[r];
    }
}

// Shared-memory layout (byte offsets, 16-byte aligned).
struct RessSmem {
    size_t pvt, diag, warp0, per_warp, bytes;
    // P_b(V) of the head [64][Bp] fp32 and the diagonal G_jj [B] f64; per warp: p [B] f64,
    // a = o . P_b(V)_j [B] f64, g = R . P_b(V)_j [B] f64 (the select's 64-bit keys before it),
    // o [64] f64, R [64] f64, hist [256] u32, kept bits [ceil(B/32)] u32
    size_t p, a, g, o, r, hist, bits;
    __host__ __device__ RessSmem(int B, int warps) {
        auto up = [](size_t x) { return (x + 15) / 16 * 16; };
        pvt = 0;
        diag = up((size_t)kDim * pv_stride(B) * 4);
        warp0 = diag + up((size_t)B * 8);
        p = 0;
        a = p + up((size_t)B * 8);
        g = a + up((size_t)B * 8);
        o = g + up((size_t)B * 8);
        r = o + kDim * 8;
        hist = r + kDim * 8;
        bits = hist + 1024;
        per_warp = up(bits + (size_t)(B + 31) / 32 * 4);
        bytes = warp0 + per_warp * warps;
    }
};

__global__ void __launch_bounds__(256)
ress_mask_kernel(Geo g, RessParams rp, const float* __restrict__ pq, const float* __restrict__ pk,
                 const float* __restrict__ pv, const double* __restrict__ G, uint32_t* __restrict__ mask_bits,
                 uint16_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int B = g.B, h = blockIdx.y;
    const int warps = blockDim.x / 32, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const RessSmem L(B, warps);
    const int Bp = pv_stride(B);
    float* pvt = reinterpret_cast<float*>(smem + L.pvt);        // [64][Bp]
    double* gdiag = reinterpret_cast<double*>(smem + L.diag);  // |P_b(V)_j|^2
    const double* Gh = G + (size_t)h * B * B;
    // stage P_b(V) of the head (already dimension-major in global memory) and G's diagonal
    const float* pvh = pv + (size_t)h * kDim * B;
    for (int x = threadIdx.x; x < kDim * B; x += blockDim.x) {
        const int e = x / B;
        pvt[e * Bp + (x - e * B)] = pvh[x];
    }
    for (int j = threadIdx.x; j < B; j += blockDim.x) gdiag[j] = Gh[(size_t)j * B + j];
    __syncthreads();
    unsigned char* ws = smem + L.warp0 + warp * L.per_warp;
    double* p = reinterpret_cast<double*>(ws + L.p);
    double* av = reinterpret_cast<double*>(ws + L.a);
    double* gv = reinterpret_cast<double*>(ws + L.g);
    uint64_t* key = reinterpret_cast<uint64_t*>(ws + L.g);     // the same array, before g
    double* o = reinterpret_cast<double*>(ws + L.o);
    double* R = reinterpret_cast<double*>(ws + L.r);
    unsigned* hist = reinterpret_cast<unsigned*>(ws + L.hist);
    uint32_t* kbits = reinterpret_cast<uint32_t*>(ws + L.bits);
    const int words = (B + 31) / 32;
    const int k = min(rp.k[h], B);
    const int i0 = blockIdx.x * rp.rows_per_cta, i1 = min(B, i0 + rp.rows_per_cta);
    const float* pkh = pk + (size_t)h * kDim * B;

    for (int i = i0 + warp; i < i1; i += warps) {
        const size_t row = (size_t)h * B + i;
        // pooled probabilities p_j (fp64 from the fp32 pooled means); R holds the pooled query
        const float* q = pq + row * kDim;
        double mx = -DBL_MAX;
        for (int e = lane; e < kDim; e += 32) R[e] = (double)__ldg(q + e);
        __syncwarp();
        for (int j = lane; j < B; j += 32) {
            float kv[kDim];   // all 64 loads in flight at once (pooled K from L2)
#pragma unroll
            for (int e = 0; e < kDim; ++e) kv[e] = __ldg(pkh + (size_t)e * B + j);
            double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
            for (int e = 0; e < kDim; e += 4) {
                s0 = fma(R[e], (double)kv[e], s0);
                s1 = fma(R[e + 1], (double)kv[e + 1], s1);
                s2 = fma(R[e + 2], (double)kv[e + 2], s2);
                s3 = fma(R[e + 3], (double)kv[e + 3], s3);
            }
            const double s = ((s0 + s1) + (s2 + s3)) * 0.125;   // 1 / sqrt(64)
            p[j] = s;
            mx = fmax(mx, s);
        }
        mx = warp_max(mx);
        double se = 0.0;
        for (int j = lane; j < B; j += 32) {
            const double e = exp(p[j] - mx);
            p[j] = e;
            se += e;
        }
        se = warp_sum(se);
        for (int j = lane; j < B; j += 32) p[j] = p[j] / se;
        __syncwarp();
        // o = sum_j p_j PV_j: lane owns dimensions lane and lane + 32
        {
            double a0 = 0.0, a1 = 0.0, b0 = 0.0, b1 = 0.0;
            const float* c0 = pvt + lane * Bp;
            const float* c1 = pvt + (lane + 32) * Bp;
            int j = 0;
            for (; j + 1 < B; j += 2) {
                a0 = fma(p[j], (double)c0[j], a0);
                b0 = fma(p[j], (double)c1[j], b0);
                a1 = fma(p[j + 1], (double)c0[j + 1], a1);
                b1 = fma(p[j + 1], (double)c1[j + 1], b1);
            }
            if (j < B) {
                a0 = fma(p[j], (double)c0[j], a0);
                b0 = fma(p[j], (double)c1[j], b0);
            }
            o[lane] = a0 + a1;
            o[lane + 32] = b0 + b1;
        }
        __syncwarp();
        double oo = fma(o[lane], o[lane], o[lane + 32] * o[lane + 32]);
        oo = warp_sum(oo);
        // a_j = o . PV_j and |delta_j|^2 = p_j^2 |o - PV_j|^2; start: the k largest (key =
        // complement of the bits of a non-negative double: smallest key = largest value)
        for (int j = lane; j < B; j += 32) {
            float pvj[kDim];
#pragma unroll
            for (int e = 0; e < kDim; ++e) pvj[e] = pvt[e * Bp + j];
            double s0 = 0.0, s1 = 0.0, t0 = 0.0, t1 = 0.0;
#pragma unroll
            for (int e = 0; e < kDim; e += 2) {
                const double d0 = o[e] - (double)pvj[e], d1 = o[e + 1] - (double)pvj[e + 1];
                s0 = fma(d0, d0, s0);
                s1 = fma(d1, d1, s1);
                t0 = fma(o[e], (double)pvj[e], t0);
                t1 = fma(o[e + 1], (double)pvj[e + 1], t1);
            }
            av[j] = t0 + t1;
            key[j] = ~(uint64_t)__double_as_longlong(p[j] * p[j] * (s0 + s1));
        }
        __syncwarp();
        warp_select_smallest(key, B, k, static_cast<uint16_t*>(nullptr), kbits, hist);
        __syncwarp();
        if (k > 0 && k < B) {
            // dropped mass and R = sum_{j dropped} delta_j
            double PD = 0.0;
            for (int j = lane; j < B; j += 32)
                if (!((kbits[j >> 5] >> (j & 31)) & 1u)) PD += p[j];
            PD = warp_sum(PD);
            {   // lane owns dimensions lane and lane + 32
                double r0 = 0.0, r1 = 0.0;
                const double o0 = o[lane], o1 = o[lane + 32];
                const float* c0 = pvt + lane * Bp;
                const float* c1 = pvt + (lane + 32) * Bp;
                for (int j = 0; j < B; ++j) {
                    if ((kbits[j >> 5] >> (j & 31)) & 1u) continue;   // kept (uniform across the warp)
                    r0 = fma(p[j], o0 - (double)c0[j], r0);
                    r1 = fma(p[j], o1 - (double)c1[j], r1);
                }
                R[lane] = r0;
                R[lane + 32] = r1;
            }
            __syncwarp();
            for (int j = lane; j < B; j += 32) gv[j] = dot_col(R, pvt, Bp, j);   // g_j = R . PV_j
            __syncwarp();
            for (int round = 0; round < rp.rounds; ++round) {
                double RR = fma(R[lane], R[lane], R[lane + 32] * R[lane + 32]);
                double Ro = fma(R[lane], o[lane], R[lane + 32] * o[lane + 32]);
                RR = warp_sum(RR);
                Ro = warp_sum(Ro);
                const double cur = RR / ((1.0 - PD) * (1.0 - PD));
                // restore: the dropped block l minimising drift(D \ {l}):
                // |R - delta_l|^2 = |R|^2 - 2 p_l (R.o - g_l) + |delta_l|^2,
                // |delta_l|^2 = p_l^2 (|o|^2 - 2 a_l + G_ll)
                ArgMin best{DBL_MAX, INT_MAX};
                for (int j = lane; j < B; j += 32) {
                    if ((kbits[j >> 5] >> (j & 31)) & 1u) continue;
                    const double dd = p[j] * p[j] * (oo - 2.0 * av[j] + gdiag[j]);
                    const double num = RR - 2.0 * p[j] * (Ro - gv[j]) + dd;
                    const double den = 1.0 - PD + p[j];
                    const double v = num / (den * den);
                    if (better(v, j, best.v, best.j)) best = {v, j};
                }
                best = warp_argmin(best.v, best.j);
                const int l = best.j;
                const double pl = p[l];
                const double* Gl = Gh + (size_t)l * B;
                // R' = R - delta_l (two dimensions per lane, kept in registers until accepted)
                const double rp0 = R[lane] - pl * (o[lane] - (double)pvt[lane * Bp + l]);
                const double rp1 = R[lane + 32] - pl * (o[lane + 32] - (double)pvt[(lane + 32) * Bp + l]);
                const double RR2 = warp_sum(fma(rp0, rp0, rp1 * rp1));
                const double Ro2 = warp_sum(fma(rp0, o[lane], rp1 * o[lane + 32]));
                const double PD2 = PD - pl;
                // drop: the kept block m != l minimising drift((D \ {l}) U {m}), with
                // R'.PV_m = g_m - p_l (a_m - G_lm)
                ArgMin bm{DBL_MAX, INT_MAX};
                for (int j = lane; j < B; j += 32) {
                    if (!((kbits[j >> 5] >> (j & 31)) & 1u) || j == l) continue;
                    const double gj = gv[j] - pl * (av[j] - Gl[j]);
                    const double dd = p[j] * p[j] * (oo - 2.0 * av[j] + gdiag[j]);
                    const double den = 1.0 - PD2 - p[j];
                    const double v = den > 0.0 ? (RR2 + 2.0 * p[j] * (Ro2 - gj) + dd) / (den * den) : DBL_MAX;
                    if (better(v, j, bm.v, bm.j)) bm = {v, j};
                }
                bm = warp_argmin(bm.v, bm.j);
                if (!(bm.v < cur) || bm.j == INT_MAX) break;       // no swap lowers the drift: stop
                const int m = bm.j;
                const double pm = p[m];
                const double* Gm = Gh + (size_t)m * B;
                R[lane] = rp0 + pm * (o[lane] - (double)pvt[lane * Bp + m]);
                R[lane + 32] = rp1 + pm * (o[lane + 32] - (double)pvt[(lane + 32) * Bp + m]);
                for (int j = lane; j < B; j += 32) gv[j] = gv[j] - pl * (av[j] - Gl[j]) + pm * (av[j] - Gm[j]);
                if (lane == 0) {
                    kbits[l >> 5] |= 1u << (l & 31);
                    kbits[m >> 5] &= ~(1u << (m & 31));
                }
                PD = PD2 + pm;
                __syncwarp();
            }
        }
        // kept blocks in ascending order
        const unsigned lt_mask = lanemask_lt();
        int pos = 0;
        for (int base = 0; base < B; base += 32) {
            const int j = base + lane;
            const bool sel = j < B && ((kbits[base >> 5] >> lane) & 1u);
            const unsigned sm = __ballot_sync(0xffffffffu, sel);
            if (sel) kv_idx[row * B + pos + __popc(sm & lt_mask)] = (uint16_t)j;
            pos += __popc(sm);
            if (mask_bits != nullptr && lane == 0) mask_bits[row * words + (base >> 5)] = sm;
        }
        if (lane == 0) kv_cnt[row] = pos;
        __syncwarp();
    }
}

}  // namespace

size_t ress_smem_bytes(int B, int warps) { return RessSmem(B, warps).bytes; }

size_t ress_workspace_bytes(const Geo& g) { return (size_t)g.H * g.B * g.B * sizeof(double); }

cudaError_t launch_ress_mask(const Geo& g, const int* k_per_head, int rounds, const float* pq, const float* pk,
                             const float* pv, void* workspace, uint32_t* mask_bits, uint16_t* kv_idx,
                             int32_t* kv_cnt, cudaStream_t st) {
    RessParams rp{};
    for (int h = 0; h < g.H; ++h) rp.k[h] = k_per_head[h];
    rp.rounds = rounds;
    double* G = static_cast<double*>(workspace);
    const dim3 ggrid((g.B + 31) / 32, (g.B + 31) / 32, g.H);
    gram_kernel<<<ggrid, 256, 0, st>>>(g.B, pv, G);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // as many warps (rows in flight) as shared memory allows, up to 8
    const size_t limit = 227 * 1024;
    int warps = 8;
    while (warps > 1 && ress_smem_bytes(g.B, warps) > limit) --warps;
    if (ress_smem_bytes(g.B, warps) > limit) return cudaErrorInvalidValue;
    // about two rounds of one CTA per SM
    const int ctas_per_head = max(1, (2 * num_sms() + g.H - 1) / g.H);
    rp.rows_per_cta = max(warps, (g.B + ctas_per_head - 1) / ctas_per_head);
    const size_t smem = ress_smem_bytes(g.B, warps);
    e = cudaFuncSetAttribute(ress_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((g.B + rp.rows_per_cta - 1) / rp.rows_per_cta, g.H);
    ress_mask_kernel<<<grid, 32 * warps, smem, st>>>(g, rp, pq, pk, pv, G, mask_bits, kv_idx, kv_cnt);
    return cudaGetLastError();
}

}  // namespace bsa
