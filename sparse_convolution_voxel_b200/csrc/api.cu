// C-ABI entry points of the convolution passes and the status helpers.
#include <cstring>

#include "common.cuh"
#include "conv_common.cuh"

namespace lat {

static bool map_ok(const lat_kmap *m) {
    if (!m || m->k3 < 1 || m->k3 > 32 || m->n_in < 0 || m->n_out < 0) return false;
    if (m->n_in >= (int64_t(1) << 31) || m->n_out >= (int64_t(1) << 31)) return false;
    if (m->n_out > 0 && (!m->nbr || !m->perm || !m->tile_mask)) return false;
    return true;
}

static bool chan_ok(int c, lat_dtype dt) {
    if (c < 8 || c % 8) return false;
    return dt == LAT_F32 ? c <= 256 : c <= 256;
}

static bool aligned16(const void *p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

template <typename F>
static lat_status by_dtype(lat_dtype dt, F &&f) {
    switch (dt) {
        case LAT_F32: return f(float{});
        case LAT_F16: return f(__half{});
        case LAT_BF16: return f(__nv_bfloat16{});
    }
    return LAT_ERR_ARG;
}

}  // namespace lat

extern "C" size_t lat_sconv_ws_bytes(int32_t op, int32_t cin, int32_t cout, const lat_kmap *map, lat_dtype dtype) {
    if (!lat::map_ok(map)) return 0;
    if (op == LAT_OP_WGRAD)
        return (dtype != LAT_F32 && lat::wgrad_tc_supported(cin, cout)) ? lat::wgrad_tc_ws_bytes(cin, cout, map)
                                                                        : lat::wgrad_simt_ws_bytes(cin, cout, map);
    // forward gathers cin channels into cout; the data gradient gathers cout into cin
    if (op == LAT_OP_FWD) return (dtype != LAT_F32 && lat::conv_tc_supported(cin, cout)) ? lat::conv_tc_ws_bytes() : 0;
    if (op == LAT_OP_DGRAD) return (dtype != LAT_F32 && lat::conv_tc_supported(cout, cin)) ? lat::conv_tc_ws_bytes() : 0;
    return 0;
}

extern "C" lat_status lat_sconv_fwd(const void *x, int32_t cin, const void *w, int32_t cout, const lat_kmap *map,
                                    void *y, lat_dtype dtype, void *ws, size_t ws_bytes, int32_t *d_status,
                                    lat_stream stream) {
    using namespace lat;
    if (!map_ok(map) || !chan_ok(cin, dtype) || !chan_ok(cout, dtype)) return LAT_ERR_ARG;
    if (map->n_out > 0 && (!y || !w || (map->n_in > 0 && !x))) return LAT_ERR_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return LAT_ERR_ARG;
    const MapView mv = make_view(map, false);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype != LAT_F32 && conv_tc_supported(cin, cout)) {
        if (!ws || ws_bytes < conv_tc_ws_bytes()) return LAT_ERR_WORKSPACE;
        return launch_conv_tc(dtype == LAT_BF16, x, cin, w, cout, map->k3, mv, false, y, ws, d_status, s);
    }
    return by_dtype(dtype, [&](auto t) {
        using T = decltype(t);
        return launch_conv_simt<T>(x, cin, w, cout, mv, false, y, d_status, s);
    });
}

extern "C" lat_status lat_sconv_dgrad(const void *dy, int32_t cout, const void *w, int32_t cin, const lat_kmap *map,
                                      int32_t flip_offsets, void *dx, lat_dtype dtype, void *ws, size_t ws_bytes,
                                      int32_t *d_status, lat_stream stream) {
    using namespace lat;
    if (!map_ok(map) || !chan_ok(cin, dtype) || !chan_ok(cout, dtype)) return LAT_ERR_ARG;
    if (flip_offsets && map->n_in != map->n_out) return LAT_ERR_ARG;
    if (map->n_out > 0 && (!dx || !w || (map->n_in > 0 && !dy))) return LAT_ERR_ARG;
    if (!aligned16(dy) || !aligned16(w) || !aligned16(dx)) return LAT_ERR_ARG;
    const MapView mv = make_view(map, flip_offsets != 0);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the pass gathers dy rows (cout channels) and produces dx rows (cin channels) with W[k]^T
    if (dtype != LAT_F32 && conv_tc_supported(cout, cin)) {
        if (!ws || ws_bytes < conv_tc_ws_bytes()) return LAT_ERR_WORKSPACE;
        return launch_conv_tc(dtype == LAT_BF16, dy, cout, w, cin, map->k3, mv, true, dx, ws, d_status, s);
    }
    return by_dtype(dtype, [&](auto t) {
        using T = decltype(t);
        return launch_conv_simt<T>(dy, cout, w, cin, mv, true, dx, d_status, s);
    });
}

extern "C" lat_status lat_sconv_wgrad(const void *x, int32_t cin, const void *dy, int32_t cout, const lat_kmap *map,
                                      float *dw, lat_dtype dtype, void *ws, size_t ws_bytes, int32_t *d_status,
                                      lat_stream stream) {
    using namespace lat;
    if (!map_ok(map) || !chan_ok(cin, dtype) || !chan_ok(cout, dtype) || !dw || !map->pair_off) return LAT_ERR_ARG;
    if (map->pair_capacity > 0 && (!map->pair_in || !map->pair_out)) return LAT_ERR_ARG;
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dw)) return LAT_ERR_ARG;
    const bool tc = dtype != LAT_F32 && wgrad_tc_supported(cin, cout);
    const size_t need = tc ? wgrad_tc_ws_bytes(cin, cout, map) : wgrad_simt_ws_bytes(cin, cout, map);
    if (ws_bytes < need || !ws) return LAT_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (tc) return launch_wgrad_tc(dtype == LAT_BF16, x, cin, dy, cout, map, dw, ws, d_status, s);
    return by_dtype(dtype, [&](auto t) {
        using T = decltype(t);
        return launch_wgrad_simt<T>(x, cin, dy, cout, map, dw, ws, d_status, s);
    });
}

extern "C" int32_t lat_status_fetch(const int32_t *d_status, lat_stream stream) {
    if (!d_status) return LAT_ERR_ARG;
    int32_t v = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, d_status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LAT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LAT_ERR_CUDA;
    return v;
}

extern "C" const char *lat_status_string(int32_t status) {
    if (status == LAT_OK) return "ok";
    if (status & LAT_ERR_ARG) return "invalid argument";
    if (status & LAT_ERR_COORD_RANGE) return "coordinate outside the packable key range";
    if (status & LAT_ERR_DUPLICATE) return "duplicate coordinate rows";
    if (status & LAT_ERR_TABLE_FULL) return "hash table full";
    if (status & LAT_ERR_CAPACITY) return "output buffer too small";
    if (status & LAT_ERR_UNSUPPORTED) return "unsupported shape or dtype";
    if (status & LAT_ERR_CUDA) return "CUDA runtime error";
    if (status & LAT_ERR_WORKSPACE) return "workspace too small";
    if (status & LAT_ERR_BAD_MAP) return "kernel map row index out of range";
    if (status & LAT_ERR_TIMEOUT) return "bounded in-kernel wait timed out";
    return "unknown status";
}

extern "C" int32_t lat_version(void) { return 100; }

extern "C" uint64_t lat_set_wait_limit_ns(uint64_t ns) { return lat::wait_limit_store().exchange(ns); }
