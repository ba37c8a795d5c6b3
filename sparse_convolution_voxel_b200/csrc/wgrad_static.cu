// Weight gradient for callers that cannot allocate device memory
// (lat_sconv_wgrad_static).
//
// Some callers cannot hand the library a scratch buffer: code that runs
// while a stream is being captured into a CUDA graph without memory nodes,
// real-time loops that forbid cudaMalloc/cudaFree (a device-wide
// synchronisation) after start-up, or hosts whose allocator is owned by
// someone else.  This entry point runs the same share-based weight-gradient
// kernels as lat_sconv_wgrad's CUDA-core path, but its scratch (the fp32
// partials of every (share, offset) segment) lives in one file-scope
// __device__ array that every GPU loading the library holds until the
// process exits.
//
// Host code must not pass the array's name to a kernel: on the host it is
// only a stand-in symbol.  Its device address is fetched per device with
// cudaGetSymbolAddress, with that device current, by the first call on that
// device that succeeds in looking it up, and kept from then on.
#include <mutex>

#include "common.cuh"
#include "conv_common.cuh"

namespace lat {
namespace {

static __device__ __align__(256) unsigned char g_wgrad_scratch[LAT_WGRAD_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // nullptr until a lookup on that device succeeded

// Device address of g_wgrad_scratch on the current device.  Only a successful
// lookup is kept; a failed one (its error cleared, so that it does not show
// up in later launch checks) is reported and tried again on the next call.
cudaError_t static_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_wgrad_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return e != cudaSuccess ? e : cudaErrorUnknown;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

bool map_ok_static(const lat_kmap *m) {
    if (!m || m->k3 < 1 || m->k3 > 32 || m->n_in < 0 || m->n_out < 0 || m->pair_capacity < 0) return false;
    if (m->n_in >= (int64_t(1) << 31) || m->n_out >= (int64_t(1) << 31)) return false;
    if (!m->pair_off || (m->pair_capacity > 0 && (!m->pair_in || !m->pair_out))) return false;
    return true;
}

}  // namespace
}  // namespace lat

extern "C" lat_status lat_sconv_wgrad_static(const void *x, int32_t cin, const void *dy, int32_t cout,
                                             const lat_kmap *map, float *dw, lat_dtype dtype, int32_t *d_status,
                                             lat_stream stream) {
    using namespace lat;
    if (!map_ok_static(map) || !dw) return LAT_ERR_ARG;
    if (cin < 8 || cin % 8 || cin > 256 || cout < 8 || cout % 8 || cout > 256) return LAT_ERR_ARG;
    if (dtype != LAT_F32 && dtype != LAT_F16 && dtype != LAT_BF16) return LAT_ERR_ARG;
    auto a16 = [](const void *p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
    if (!a16(x) || !a16(dy) || !a16(dw)) return LAT_ERR_ARG;
    // every byte of scratch this call reads is written earlier in the same call,
    // so nothing left over from a previous call needs clearing; every check
    // comes before the first launch
    if (wgrad_simt_ws_bytes(cin, cout, map) > size_t(LAT_WGRAD_STATIC_SCRATCH_BYTES)) return LAT_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (static_scratch(&scratch) != cudaSuccess) return LAT_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (dtype) {
        case LAT_F32: return launch_wgrad_simt<float>(x, cin, dy, cout, map, dw, scratch, d_status, s);
        case LAT_F16: return launch_wgrad_simt<__half>(x, cin, dy, cout, map, dw, scratch, d_status, s);
        case LAT_BF16: return launch_wgrad_simt<__nv_bfloat16>(x, cin, dy, cout, map, dw, scratch, d_status, s);
    }
    return LAT_ERR_ARG;
}
