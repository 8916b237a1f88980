// C ABI of the block-sparse global attention library: host-side validation, per-head
// block budgets, and stream-ordered launches of the device steps. The library owns no
// device memory; every buffer comes from the caller.
#include <cmath>
#include <cstdint>
#include <cstdio>

#include "common.cuh"
#include "tc_layout.cuh"

namespace bsa {

int num_sms() {
    static int cached = 0;
    if (cached == 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            cached = n;
        else
            return 148;
    }
    return cached;
}

cudaError_t launch_attn_tc(const Geo& g, int mode, const void* ws, const uint16_t* kv_idx,
                           const int32_t* kv_cnt, float* o_part, float* lse_part, void* out,
                           int32_t* status, cudaStream_t st);
cudaError_t launch_pack_pool(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                             float* pq, float* pk, int32_t* status, cudaStream_t st);
cudaError_t launch_pack(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                        int32_t* status, cudaStream_t st);
cudaError_t launch_random_mask(const Geo& g, const int* k_per_head, uint64_t seed, uint32_t* mask_bits,
                               uint16_t* kv_idx, int32_t* kv_cnt, cudaStream_t st);
cudaError_t launch_uniform_mask(const Geo& g, int stride, uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                                cudaStream_t st);
cudaError_t launch_probe_mask(const Geo& g, const int* k_per_head, const float* pq, const float* pk,
                              uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt, cudaStream_t st);
cudaError_t launch_gemm_bf16(int M, int N, int K, const void* a, const void* b, const float* bias,
                             void* const out[3], int split, int32_t* status, cudaStream_t st);
cudaError_t launch_pack_frames(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                               int32_t* status, cudaStream_t st);
cudaError_t launch_attn_frame(const Geo& g, const void* ws, void* out, int32_t* status, cudaStream_t st);
cudaError_t launch_pool_v(const Geo& g, bsa_dtype dt, const void* v, float* pv, cudaStream_t st);
size_t ress_smem_bytes(int B, int warps);
size_t ress_workspace_bytes(const Geo& g);
cudaError_t launch_ress_mask(const Geo& g, const int* k_per_head, int rounds, const float* pq, const float* pk,
                             const float* pv, void* workspace, uint32_t* mask_bits, uint16_t* kv_idx,
                             int32_t* kv_cnt, cudaStream_t st);

namespace {

constexpr double kTieEps = 1e-9;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bsa_status make_geo(const bsa_layout* L, Geo* g) {
    if (L == nullptr) return BSA_ERR_INVALID_ARG;
    if (L->frames < 1 || L->tokens_per_frame < 1 || L->special_per_frame < 0 ||
        L->special_per_frame >= L->tokens_per_frame || L->heads < 1 || L->block < 1 ||
        L->head_dim < 1 || (L->dtype != BSA_F32 && L->dtype != BSA_BF16))
        return BSA_ERR_INVALID_ARG;
    if (L->head_dim != BSA_HEAD_DIM || L->heads > BSA_MAX_HEADS) return BSA_ERR_UNSUPPORTED;
    const int64_t N = (int64_t)L->frames * L->tokens_per_frame;
    if (N > (int64_t)INT32_MAX / 2) return BSA_ERR_UNSUPPORTED;
    g->F = L->frames;
    g->T = L->tokens_per_frame;
    g->S = L->special_per_frame;
    g->H = L->heads;
    g->d = L->head_dim;
    g->b = L->block;
    g->P = g->T - g->S;
    g->N = (int)N;
    g->Np = g->F * g->P;
    g->Ns = g->F * g->S;
    g->B = (int)(((int64_t)g->Np + g->b - 1) / g->b);
    if (g->B > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
    if (L->dtype == BSA_F32 && g->N > BSA_F32_MAX_TOKENS) return BSA_ERR_UNSUPPORTED;
    return BSA_OK;
}

bsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

int k_rho(int B, double rho) { return (int)std::floor(B * (1.0 - rho) + kTieEps); }

int k_density(int B, double d) {
    int k = (int)std::floor(B * d + kTieEps);
    return k < 1 ? 1 : (k > B ? B : k);
}

// The tensor-core path tiles the packed patch rows in 128-row query tiles and key tiles
// of b rows.
bool tc_supported(const Geo& g) { return g.b == 64 || g.b == 128; }

bool aligned1024(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1023u) == 0; }

// Per-head block budgets: k = floor(B (1 - rho)) for every head, or k_h from the per-head
// densities, whose sum must be the layer budget H (1 - rho).
bsa_status head_budgets_k(const Geo& g, double rho, const double* head_density, int* k) {
    if (!(rho >= 0.0 && rho <= 1.0)) return BSA_ERR_INVALID_ARG;
    if (head_density == nullptr) {
        const int kk = k_rho(g.B, rho);
        for (int h = 0; h < g.H; ++h) k[h] = kk;
        return BSA_OK;
    }
    double sum = 0.0;
    for (int h = 0; h < g.H; ++h) {
        if (!(head_density[h] >= 0.0 && head_density[h] <= 1.0)) return BSA_ERR_INVALID_ARG;
        sum += head_density[h];
        k[h] = k_density(g.B, head_density[h]);
    }
    if (std::fabs(sum - g.H * (1.0 - rho)) > 1e-9 * g.H) return BSA_ERR_INVALID_ARG;
    return BSA_OK;
}

// Output buffers of a block selector: the lists, counts and optional bits.
bool lists_ok(const uint16_t* kv_idx, const int32_t* kv_cnt, const uint32_t* mask_bits) {
    return kv_idx && kv_cnt && aligned16(kv_idx) && aligned16(kv_cnt) && (!mask_bits || aligned16(mask_bits));
}

bsa_status check_ws(const Geo& g, const void* ws, size_t bytes) {
    if (ws == nullptr || !aligned1024(ws)) return BSA_ERR_INVALID_ARG;
    if (bytes < packed_layout(g).bytes) return BSA_ERR_INVALID_ARG;
    return BSA_OK;
}

}  // namespace

// Layout validation for entry points defined in other files.
bsa_status make_geo_checked(const bsa_layout* L, Geo* g) { return make_geo(L, g); }

}  // namespace bsa

using namespace bsa;

extern "C" {

const char* bsa_status_string(bsa_status s) {
    switch (s) {
        case BSA_OK: return "ok";
        case BSA_ERR_INVALID_ARG: return "invalid argument";
        case BSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case BSA_ERR_CUDA: return "CUDA error";
        case BSA_ERR_TIMEOUT: return "device wait timed out";
        case BSA_ERR_DEVICE_BOUNDS: return "device index out of range";
        case BSA_ERR_RANGE: return "input value outside the range of the kernels' operand type";
    }
    return "unknown status";
}

bsa_status bsa_num_blocks(const bsa_layout* layout, int32_t* num_blocks) {
    if (num_blocks == nullptr) return BSA_ERR_INVALID_ARG;
    Geo g;
    const bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    *num_blocks = g.B;
    return BSA_OK;
}

bsa_status bsa_workspace_size(const bsa_layout* layout, size_t* bytes) {
    if (bytes == nullptr) return BSA_ERR_INVALID_ARG;
    Geo g;
    const bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    *bytes = layout->dtype == BSA_BF16 ? packed_layout(g).bytes : 0;
    return BSA_OK;
}

bsa_status bsa_pack_qkv(const bsa_layout* layout, const void* q, const void* k, const void* v,
                        void* workspace, size_t workspace_bytes, int32_t* status_dev,
                        bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16) return BSA_OK;
    if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return BSA_ERR_INVALID_ARG;
    s = check_ws(g, workspace, workspace_bytes);
    if (s != BSA_OK) return s;
    return from_cuda(launch_pack(g, q, k, v, workspace, status_dev, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_pack_pool_qkv(const bsa_layout* layout, const void* q, const void* k, const void* v,
                             void* workspace, size_t workspace_bytes, float* pq, float* pk,
                             int32_t* status_dev, bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!q || !k || !pq || !pk) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(pq) || !aligned16(pk)) return BSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (layout->dtype != BSA_BF16) return from_cuda(launch_pool(g, layout->dtype, q, k, pq, pk, st));
    if (!v || !aligned16(v)) return BSA_ERR_INVALID_ARG;
    s = check_ws(g, workspace, workspace_bytes);
    if (s != BSA_OK) return s;
    if (!tc_supported(g)) {   // the one-pass kernel needs whole blocks per 128-row tile
        cudaError_t e = launch_pack(g, q, k, v, workspace, status_dev, st);
        if (e == cudaSuccess) e = launch_pool(g, layout->dtype, q, k, pq, pk, st);
        return from_cuda(e);
    }
    return from_cuda(launch_pack_pool(g, q, k, v, workspace, pq, pk, status_dev, st));
}

bsa_status bsa_k_from_rho(int32_t num_blocks, double rho, int32_t* k) {
    if (k == nullptr || num_blocks < 1 || !(rho >= 0.0 && rho <= 1.0)) return BSA_ERR_INVALID_ARG;
    *k = k_rho(num_blocks, rho);
    return BSA_OK;
}

bsa_status bsa_k_from_density(int32_t num_blocks, double density, int32_t* k) {
    if (k == nullptr || num_blocks < 1 || !(density >= 0.0 && density <= 1.0)) return BSA_ERR_INVALID_ARG;
    *k = k_density(num_blocks, density);
    return BSA_OK;
}

bsa_status bsa_head_budgets(const double* scores, int32_t heads, double rho, double cap,
                            double* density) {
    if (scores == nullptr || density == nullptr || heads < 1 || heads > BSA_MAX_HEADS ||
        !(rho >= 0.0 && rho <= 1.0) || !(cap > 0.0))
        return BSA_ERR_INVALID_ARG;
    const double total = heads * (1.0 - rho);
    if (total > heads * cap + 1e-12) return BSA_ERR_INVALID_ARG;
    for (int h = 0; h < heads; ++h)
        if (!(scores[h] > 0.0) || !std::isfinite(scores[h])) return BSA_ERR_INVALID_ARG;
    bool capped[BSA_MAX_HEADS] = {false};
    for (int round = 0; round <= heads; ++round) {
        int ncap = 0;
        double sfree = 0.0;
        for (int h = 0; h < heads; ++h) {
            if (capped[h]) ++ncap;
            else sfree += scores[h];
        }
        if (ncap == heads) {
            for (int h = 0; h < heads; ++h) density[h] = cap;
            break;
        }
        const double remaining = total - cap * ncap;
        bool newly = false;
        for (int h = 0; h < heads; ++h) {
            density[h] = capped[h] ? cap : remaining * scores[h] / sfree;
            if (!capped[h] && density[h] > cap) newly = true;
        }
        if (!newly) break;
        for (int h = 0; h < heads; ++h)
            if (!capped[h] && density[h] > cap) capped[h] = true;
    }
    return BSA_OK;
}

bsa_status bsa_selftest_wait_timeout(int32_t* status_dev, uint32_t limit_us, bsa_stream_t stream) {
    if (status_dev == nullptr || (reinterpret_cast<uintptr_t>(status_dev) & 3u) != 0u || limit_us < 1u ||
        limit_us > 10000000u)
        return BSA_ERR_INVALID_ARG;
    return from_cuda(launch_wait_timeout(status_dev, (uint64_t)limit_us * 1000ull,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_check_status(int32_t* status_dev, bsa_stream_t stream) {
    if (status_dev == nullptr) return BSA_ERR_INVALID_ARG;
    int32_t v = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, status_dev, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return BSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BSA_ERR_CUDA;
    if (v != 0 && cudaMemsetAsync(status_dev, 0, sizeof(int32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
    if (v == 0) return BSA_OK;
    if (v == BSA_ERR_TIMEOUT || v == BSA_ERR_DEVICE_BOUNDS || v == BSA_ERR_RANGE) return (bsa_status)v;
    return BSA_ERR_CUDA;
}

bsa_status bsa_pool_qk(const bsa_layout* layout, const void* q, const void* k, float* pq,
                       float* pk, int32_t* status_dev, bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!q || !k || !pq || !pk) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(pq) || !aligned16(pk)) return BSA_ERR_INVALID_ARG;
    return from_cuda(launch_pool(g, layout->dtype, q, k, pq, pk, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_predict_mask(const bsa_layout* layout, const float* pq, const float* pk, double rho,
                            double tau, const double* head_density, uint32_t* mask_bits,
                            uint16_t* kv_idx, int32_t* kv_cnt, int32_t* status_dev,
                            bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!pq || !pk || !kv_idx || !kv_cnt) return BSA_ERR_INVALID_ARG;
    if (!aligned16(pq) || !aligned16(pk) || !aligned16(kv_idx) || !aligned16(kv_cnt) ||
        (mask_bits && !aligned16(mask_bits)))
        return BSA_ERR_INVALID_ARG;
    if (!(tau >= 0.0 && tau <= 1.0)) return BSA_ERR_INVALID_ARG;
    if (g.B > 65535) return BSA_ERR_UNSUPPORTED;
    MaskParams mp;
    mp.tau = tau;
    if ((s = head_budgets_k(g, rho, head_density, mp.k)) != BSA_OK) return s;
    return from_cuda(launch_mask(g, mp, pq, pk, mask_bits, kv_idx, kv_cnt, status_dev,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_random_mask(const bsa_layout* layout, double rho, const double* head_density, uint64_t seed,
                           uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt, int32_t* status_dev,
                           bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!lists_ok(kv_idx, kv_cnt, mask_bits)) return BSA_ERR_INVALID_ARG;
    if (g.B > 65535) return BSA_ERR_UNSUPPORTED;
    int k[BSA_MAX_HEADS];
    if ((s = head_budgets_k(g, rho, head_density, k)) != BSA_OK) return s;
    return from_cuda(launch_random_mask(g, k, seed, mask_bits, kv_idx, kv_cnt, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_uniform_mask(const bsa_layout* layout, int32_t stride, uint32_t* mask_bits, uint16_t* kv_idx,
                            int32_t* kv_cnt, int32_t* status_dev, bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (stride < 1 || !lists_ok(kv_idx, kv_cnt, mask_bits)) return BSA_ERR_INVALID_ARG;
    if (g.B > 65535) return BSA_ERR_UNSUPPORTED;
    return from_cuda(launch_uniform_mask(g, stride, mask_bits, kv_idx, kv_cnt, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_probe_mask(const bsa_layout* layout, const float* pq, const float* pk, double rho,
                          const double* head_density, uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt,
                          int32_t* status_dev, bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!pq || !pk || !aligned16(pq) || !aligned16(pk) || !lists_ok(kv_idx, kv_cnt, mask_bits))
        return BSA_ERR_INVALID_ARG;
    if (g.B > 65535) return BSA_ERR_UNSUPPORTED;
    int k[BSA_MAX_HEADS];
    if ((s = head_budgets_k(g, rho, head_density, k)) != BSA_OK) return s;
    return from_cuda(launch_probe_mask(g, k, pq, pk, mask_bits, kv_idx, kv_cnt, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_block_sparse_attn(const bsa_layout* layout, const void* q, const void* k,
                                 const void* v, const void* workspace, size_t workspace_bytes,
                                 const uint16_t* kv_idx, const int32_t* kv_cnt,
                                 float* o_pp, float* lse_pp, int32_t* status_dev,
                                 bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!q || !k || !v || !kv_idx || !kv_cnt || !o_pp || !lse_pp) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_pp) || !aligned16(lse_pp) ||
        !aligned16(kv_idx) || !aligned16(kv_cnt))
        return BSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (layout->dtype == BSA_BF16) {
        if (!tc_supported(g)) return BSA_ERR_UNSUPPORTED;
        s = check_ws(g, workspace, workspace_bytes);
        if (s != BSA_OK) return s;
        return from_cuda(launch_attn_tc(g, 0, workspace, kv_idx, kv_cnt, o_pp, lse_pp, nullptr, status_dev, st));
    }
    return from_cuda(launch_attn_simt(g, BSA_F32, 0, q, k, v, kv_idx, kv_cnt, o_pp, lse_pp, nullptr,
                                      status_dev, st));
}

bsa_status bsa_special_dense(const bsa_layout* layout, const void* q, const void* k, const void* v,
                             const void* workspace, size_t workspace_bytes, void* out, float* o_ps,
                             float* lse_ps, int32_t* status_dev, bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!q || !k || !v || !out || (o_ps && !lse_ps)) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (o_ps && (!aligned16(o_ps) || !aligned16(lse_ps))))
        return BSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool tc = layout->dtype == BSA_BF16;
    if (tc && !tc_supported(g)) return BSA_ERR_UNSUPPORTED;
    if (tc && (s = check_ws(g, workspace, workspace_bytes)) != BSA_OK) return s;
    cudaError_t e = cudaSuccess;
    if (g.Ns > 0) {
        e = tc ? launch_attn_tc(g, 2, workspace, nullptr, nullptr, nullptr, nullptr, out, status_dev, st)
               : launch_attn_simt(g, BSA_F32, 2, q, k, v, nullptr, nullptr, nullptr, nullptr, out, status_dev, st);
        if (e != cudaSuccess) return BSA_ERR_CUDA;
    }
    if (o_ps != nullptr) {
        if (g.Ns == 0) {   // no special keys: empty partial (o = 0, lse = -inf)
            e = launch_fill(o_ps, (size_t)g.Np * g.H * g.d, 0.f, st);
            if (e == cudaSuccess) e = launch_fill(lse_ps, (size_t)g.H * g.Np, -INFINITY, st);
        } else {
            e = tc ? launch_attn_tc(g, 1, workspace, nullptr, nullptr, o_ps, lse_ps, nullptr, status_dev, st)
                   : launch_attn_simt(g, BSA_F32, 1, q, k, v, nullptr, nullptr, o_ps, lse_ps, nullptr, status_dev, st);
        }
    }
    return from_cuda(e);
}

bsa_status bsa_block_sparse_attn_fused(const bsa_layout* layout, const void* q, const void* k, const void* v,
                                       const void* workspace, size_t workspace_bytes, const uint16_t* kv_idx,
                                       const int32_t* kv_cnt, void* out, int32_t* status_dev,
                                       bsa_stream_t stream) {
    (void)q;
    (void)k;
    (void)v;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16 || !tc_supported(g)) return BSA_ERR_UNSUPPORTED;
    if (!kv_idx || !kv_cnt || !out || !aligned16(out) || !aligned16(kv_idx) || !aligned16(kv_cnt))
        return BSA_ERR_INVALID_ARG;
    s = check_ws(g, workspace, workspace_bytes);
    if (s != BSA_OK) return s;
    return from_cuda(launch_attn_tc(g, 3, workspace, kv_idx, kv_cnt, nullptr, nullptr, out, status_dev,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_pool_v(const bsa_layout* layout, const void* v, float* pv, int32_t* status_dev, bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!v || !pv || !aligned16(v) || !aligned16(pv)) return BSA_ERR_INVALID_ARG;
    return from_cuda(launch_pool_v(g, layout->dtype, v, pv, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_ress_workspace_size(const bsa_layout* layout, size_t* bytes) {
    if (bytes == nullptr) return BSA_ERR_INVALID_ARG;
    Geo g;
    const bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    *bytes = ress_workspace_bytes(g);
    return BSA_OK;
}

bsa_status bsa_ress_mask(const bsa_layout* layout, const float* pq, const float* pk, const float* pv, double rho,
                         const double* head_density, int32_t rounds, void* workspace, size_t workspace_bytes,
                         uint32_t* mask_bits, uint16_t* kv_idx, int32_t* kv_cnt, int32_t* status_dev,
                         bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!pq || !pk || !pv || !aligned16(pq) || !aligned16(pk) || !aligned16(pv) || !lists_ok(kv_idx, kv_cnt, mask_bits))
        return BSA_ERR_INVALID_ARG;
    if (rounds < 0 || rounds > BSA_RESS_MAX_ROUNDS) return BSA_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < ress_workspace_bytes(g))
        return BSA_ERR_INVALID_ARG;
    if (ress_smem_bytes(g.B, 1) > 227u * 1024u) return BSA_ERR_UNSUPPORTED;
    int k[BSA_MAX_HEADS];
    if ((s = head_budgets_k(g, rho, head_density, k)) != BSA_OK) return s;
    return from_cuda(launch_ress_mask(g, k, rounds, pq, pk, pv, workspace, mask_bits, kv_idx, kv_cnt,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_qkv_project(const bsa_layout* layout, const void* x, const void* w_qkv, const float* b_qkv,
                           void* q, void* k, void* v, int32_t* status_dev, bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    if (!x || !w_qkv || !q || !k || !v) return BSA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        (b_qkv && !aligned16(b_qkv)))
        return BSA_ERR_INVALID_ARG;
    const int C = g.H * g.d;
    void* const outs[3] = {q, k, v};
    return from_cuda(launch_gemm_bf16(g.N, 3 * C, C, x, w_qkv, b_qkv, outs, C, status_dev,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_out_project(const bsa_layout* layout, const void* o, const void* w_o, const float* b_o, void* y,
                           int32_t* status_dev, bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    if (!o || !w_o || !y || !aligned16(o) || !aligned16(w_o) || !aligned16(y) || (b_o && !aligned16(b_o)))
        return BSA_ERR_INVALID_ARG;
    const int C = g.H * g.d;
    void* const outs[3] = {y, y, y};
    return from_cuda(launch_gemm_bf16(g.N, C, C, o, w_o, b_o, outs, C, status_dev,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_frame_workspace_size(const bsa_layout* layout, size_t* bytes) {
    if (bytes == nullptr) return BSA_ERR_INVALID_ARG;
    Geo g;
    const bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    *bytes = layout->dtype == BSA_BF16 ? frame_layout(g).bytes : 0;
    return BSA_OK;
}

bsa_status bsa_pack_frames(const bsa_layout* layout, const void* q, const void* k, const void* v,
                           void* workspace, size_t workspace_bytes, int32_t* status_dev, bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return BSA_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned1024(workspace) || workspace_bytes < frame_layout(g).bytes)
        return BSA_ERR_INVALID_ARG;
    return from_cuda(launch_pack_frames(g, q, k, v, workspace, status_dev, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_frame_attention(const bsa_layout* layout, const void* workspace, size_t workspace_bytes, void* out,
                               int32_t* status_dev, bsa_stream_t stream) {
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    if (!out || !aligned16(out)) return BSA_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned1024(workspace) || workspace_bytes < frame_layout(g).bytes)
        return BSA_ERR_INVALID_ARG;
    return from_cuda(launch_attn_frame(g, workspace, out, status_dev, reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_merge(const bsa_layout* layout, const float* o_pp, const float* lse_pp,
                     const float* o_ps, const float* lse_ps, void* out, int32_t* status_dev,
                     bsa_stream_t stream) {
    (void)status_dev;
    Geo g;
    bsa_status s = make_geo(layout, &g);
    if (s != BSA_OK) return s;
    if (!o_pp || !lse_pp || !o_ps || !lse_ps || !out) return BSA_ERR_INVALID_ARG;
    if (!aligned16(o_pp) || !aligned16(o_ps) || !aligned16(out) || !aligned16(lse_pp) || !aligned16(lse_ps))
        return BSA_ERR_INVALID_ARG;
    return from_cuda(launch_merge(g, layout->dtype, o_pp, lse_pp, o_ps, lse_ps, out,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
