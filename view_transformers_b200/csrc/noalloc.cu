// Allocation-free variant of the bf16 attention steps. The packed copy of Q, K and V and
// the partial results of the special queries live in one file-scope device array instead
// of a caller-provided workspace, so a caller that cannot allocate device memory can still
// run the layer: for example code inside a host framework whose memory pool owns every
// device allocation, or a latency-critical loop where cudaMalloc/cudaFree are not allowed
// because they can synchronize the device.
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "tc_layout.cuh"

namespace bsa {
cudaError_t launch_attn_tc(const Geo& g, int mode, const void* ws, const uint16_t* kv_idx,
                           const int32_t* kv_cnt, float* o_part, float* lse_part, void* out,
                           int32_t* status, cudaStream_t st);
cudaError_t launch_pack(const Geo& g, const void* q, const void* k, const void* v, void* ws,
                        int32_t* status, cudaStream_t st);
bsa_status make_geo_checked(const bsa_layout* L, Geo* g);
}  // namespace bsa

namespace {

// Shared by every call on a device and kept until the process exits; +1 KB so that the
// packed tiles can start on a 1024-byte boundary inside it.
static __device__ __align__(256) unsigned char g_scratch[BSA_NOALLOC_SCRATCH_BYTES + 1024];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_dev[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_dev[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = p;
    }
    *out = g_scratch_dev[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" bsa_status bsa_attention_noalloc(const bsa_layout* layout, const void* q, const void* k,
                                            const void* v, const uint16_t* kv_idx, const int32_t* kv_cnt,
                                            void* out, int32_t* status_dev, bsa_stream_t stream) {
    using namespace bsa;
    Geo g;
    bsa_status s = make_geo_checked(layout, &g);
    if (s != BSA_OK) return s;
    if (layout->dtype != BSA_BF16 || !(g.b == 64 || g.b == 128)) return BSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !kv_idx || !kv_cnt || !out) return BSA_ERR_INVALID_ARG;
    const uintptr_t a = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) |
                        reinterpret_cast<uintptr_t>(kv_idx) | reinterpret_cast<uintptr_t>(kv_cnt);
    if (a & 15u) return BSA_ERR_INVALID_ARG;
    if (packed_layout(g).bytes > BSA_NOALLOC_SCRATCH_BYTES) return BSA_ERR_UNSUPPORTED;
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return BSA_ERR_CUDA;
    void* ws = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(base) + 1023) & ~uintptr_t(1023));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (launch_pack(g, q, k, v, ws, status_dev, st) != cudaSuccess) return BSA_ERR_CUDA;
    if (g.Ns > 0 &&
        launch_attn_tc(g, 2, ws, nullptr, nullptr, nullptr, nullptr, out, status_dev, st) != cudaSuccess)
        return BSA_ERR_CUDA;
    if (launch_attn_tc(g, 3, ws, kv_idx, kv_cnt, nullptr, nullptr, out, status_dev, st) != cudaSuccess)
        return BSA_ERR_CUDA;
    return BSA_OK;
}
