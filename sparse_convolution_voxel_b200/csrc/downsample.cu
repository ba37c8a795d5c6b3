// Output-support generation of a strided Conv3d (lat_downsample_ws_bytes,
// lat_downsample_coords).
//
// Torch Lattice docs, "Migrating from TorchSparse", "Convolution mapping":
// a strided forward convolution creates a downsampled support.  The coarse
// support is every q whose window {stride*q + off - pad, off in [0,K)^3}
// holds an active input.  Each input row proposes the coarse rows whose
// windows contain it (exactly one when K == stride and pad == 0: floor(p/s)),
// the packed keys are radix sorted and made unique, so the result is in
// canonical (b, x, y, z) order and independent of the input row order.
#include <cub/device/device_radix_sort.cuh>
#include <cub/device/device_select.cuh>

#include "common.cuh"

namespace lat {

struct DownGeom {
    int ks[3], st[3], pd[3];
    int per_axis[3];  // ceil(K/s): candidate offsets per axis
    int cands;        // product of per_axis
};

__global__ void __launch_bounds__(256)
down_candidates_kernel(const int4 *__restrict__ coords, int64_t n, DownGeom g, uint64_t *__restrict__ keys,
                       int32_t *d_status) {
    const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (i >= n) return;
    const int4 c = __ldg(coords + i);
    uint64_t self;
    uint64_t *dst = keys + i * g.cands;
    if (!pack_key(c.x, c.y, c.z, c.w, self)) {
        for (int e = 0; e < g.cands; ++e) dst[e] = kEmptyKey;
        flag(d_status, LAT_ERR_COORD_RANGE);
        return;
    }
    const int p[3] = {c.y, c.z, c.w};
    int first[3];  // smallest off in [0,K) with (p - off + pad) divisible by s
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const int r = (p[a] + g.pd[a]) - floordiv(p[a] + g.pd[a], g.st[a]) * g.st[a];
        first[a] = r;
    }
    int e = 0;
    for (int u = 0; u < g.per_axis[0]; ++u)
        for (int v = 0; v < g.per_axis[1]; ++v)
            for (int w = 0; w < g.per_axis[2]; ++w, ++e) {
                const int off[3] = {first[0] + u * g.st[0], first[1] + v * g.st[1], first[2] + w * g.st[2]};
                uint64_t key = kEmptyKey;
                bool ok = off[0] < g.ks[0] && off[1] < g.ks[1] && off[2] < g.ks[2];
                if (ok) {
                    int q[3];
#pragma unroll
                    for (int a = 0; a < 3; ++a) q[a] = (p[a] - off[a] + g.pd[a]) / g.st[a];  // exact division
                    if (!pack_key(c.x, q[0], q[1], q[2], key)) key = kEmptyKey;
                }
                dst[e] = key;
            }
}

// Unpack the unique keys (the last one may be the EMPTY filler) into coordinate rows.
__global__ void __launch_bounds__(256)
down_unpack_kernel(const uint64_t *__restrict__ uniq, const int *__restrict__ n_uniq, int4 *__restrict__ out,
                   int64_t capacity, int64_t *__restrict__ n_out_dev) {
    const int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    int64_t m = *n_uniq;
    if (m > 0 && uniq[m - 1] == kEmptyKey) --m;
    if (r == 0) *n_out_dev = m;
    if (r >= m || r >= capacity) return;
    int4 c;
    unpack_key(uniq[r], c);
    out[r] = c;
}

struct DownWs {
    uint64_t *keys, *sorted, *uniq;
    int *n_uniq;
    int64_t *n_out_dev;
    void *sort_tmp, *sel_tmp;
    size_t sort_bytes, sel_bytes, total;
};

static bool down_geom(const lat_geom *geom, DownGeom &g) {
    if (!geom || geom->mode != LAT_STRIDED) return false;
    g.cands = 1;
    for (int a = 0; a < 3; ++a) {
        if (geom->ksize[a] < 1 || geom->stride[a] < 1 || geom->pad[a] < 0 || geom->pad[a] >= geom->ksize[a] + 32768)
            return false;
        g.ks[a] = geom->ksize[a];
        g.st[a] = geom->stride[a];
        g.pd[a] = geom->pad[a];
        g.per_axis[a] = (geom->ksize[a] + geom->stride[a] - 1) / geom->stride[a];
        g.cands *= g.per_axis[a];
    }
    return g.ks[0] * g.ks[1] * g.ks[2] <= 32;
}

static DownWs carve_down_ws(void *base, int64_t n_items) {
    DownWs w{};
    Carver cv(base);
    w.keys = cv.take<uint64_t>(size_t(n_items));
    w.sorted = cv.take<uint64_t>(size_t(n_items));
    w.uniq = cv.take<uint64_t>(size_t(n_items));
    w.n_uniq = cv.take<int>(1);
    w.n_out_dev = cv.take<int64_t>(1);
    cub::DeviceRadixSort::SortKeys(nullptr, w.sort_bytes, (const uint64_t *)nullptr, (uint64_t *)nullptr,
                                   int(n_items), 0, 64);
    cub::DeviceSelect::Unique(nullptr, w.sel_bytes, (const uint64_t *)nullptr, (uint64_t *)nullptr, (int *)nullptr,
                              int(n_items));
    w.sort_tmp = cv.take<char>(w.sort_bytes);
    w.sel_tmp = cv.take<char>(w.sel_bytes);
    w.total = align_up(cv.used, 256);
    return w;
}

}  // namespace lat

extern "C" size_t lat_downsample_ws_bytes(int64_t n_in, const lat_geom *geom) {
    lat::DownGeom g;
    if (n_in < 0 || !lat::down_geom(geom, g)) return 0;
    const int64_t items = n_in * g.cands;
    if (items >= (int64_t(1) << 31)) return 0;
    return lat::carve_down_ws(nullptr, items).total;
}

extern "C" lat_status lat_downsample_coords(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                                            int32_t *out_coords, int64_t out_capacity, int64_t *n_out, void *ws,
                                            size_t ws_bytes, int32_t *d_status, lat_stream stream) {
    using namespace lat;
    DownGeom g;
    if (!n_out || n_in < 0 || out_capacity < 0 || !down_geom(geom, g)) return LAT_ERR_ARG;
    if (n_in > 0 && (!coords || (out_capacity > 0 && !out_coords))) return LAT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(coords) % 16 || reinterpret_cast<uintptr_t>(out_coords) % 16) return LAT_ERR_ARG;
    const int64_t items = n_in * g.cands;
    if (items >= (int64_t(1) << 31)) return LAT_ERR_UNSUPPORTED;
    *n_out = 0;
    if (n_in == 0) return LAT_OK;
    const DownWs need = carve_down_ws(nullptr, items);
    if (!ws || ws_bytes < need.total) return LAT_ERR_WORKSPACE;
    DownWs w = carve_down_ws(ws, items);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    down_candidates_kernel<<<unsigned((n_in + 255) / 256), 256, 0, s>>>(reinterpret_cast<const int4 *>(coords), n_in,
                                                                         g, w.keys, d_status);
    LAT_CUDA_TRY(cudaGetLastError());
    size_t b = w.sort_bytes;
    LAT_CUDA_TRY(cub::DeviceRadixSort::SortKeys(w.sort_tmp, b, w.keys, w.sorted, int(items), 0, 64, s));
    b = w.sel_bytes;
    LAT_CUDA_TRY(cub::DeviceSelect::Unique(w.sel_tmp, b, w.sorted, w.uniq, w.n_uniq, int(items), s));
    down_unpack_kernel<<<unsigned((items + 255) / 256), 256, 0, s>>>(w.uniq, w.n_uniq,
                                                                     reinterpret_cast<int4 *>(out_coords),
                                                                     out_capacity, w.n_out_dev);
    LAT_CUDA_TRY(cudaGetLastError());
    int64_t m = 0;
    LAT_CUDA_TRY(cudaMemcpyAsync(&m, w.n_out_dev, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    LAT_CUDA_TRY(cudaStreamSynchronize(s));
    *n_out = m;
    return m > out_capacity ? LAT_ERR_CAPACITY : LAT_OK;
}
