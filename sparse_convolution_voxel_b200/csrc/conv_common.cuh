// Kernel-map view shared by the convolution kernels.
#pragma once

#include <algorithm>

#include "common.cuh"

namespace lat {

// Read-only view of a lat_kmap as one convolution pass consumes it.
// flip: the pass walks the map backwards (data gradient of a submanifold
// convolution): slot k of output row i reads nbr[k3-1-k][i], and a tile's
// offset set is the bit-reversed forward set.
struct MapView {
    const int32_t *nbr;
    const int32_t *perm;
    const uint32_t *tile_mask;
    int64_t n_in;   // rows of the gathered operand
    int64_t n_out;  // rows written (== leading dimension of nbr)
    int64_t ntiles;
    int k3;
    int flip;
    int centre;  // submanifold maps: the centre offset, whose neighbour of row j is j itself; else -1

    // a stored tile mask as this pass sees it (bits past the offset count dropped)
    __device__ __forceinline__ uint32_t flip_mask(uint32_t m) const {
        m &= k3 >= 32 ? 0xFFFFFFFFu : ((1u << k3) - 1u);
        return flip ? (__brev(m) >> (32 - k3)) : m;
    }
    __device__ __forceinline__ uint32_t tile_mask_at(int64_t t) const { return flip_mask(tile_mask[t]); }
    __device__ __forceinline__ const int32_t *neighbour_ptr(int k, int64_t j) const {
        const int kk = flip ? (k3 - 1 - k) : k;
        return nbr + int64_t(kk) * n_out + j;
    }
    __device__ __forceinline__ int neighbour(int k, int64_t j) const {
        if (k == centre) return int(j);
        const int kk = flip ? (k3 - 1 - k) : k;
        return __ldg(nbr + int64_t(kk) * n_out + j);
    }
};

inline MapView make_view(const lat_kmap *m, bool flip) {
    MapView v{};
    v.nbr = m->nbr;
    v.perm = m->perm;
    v.tile_mask = m->tile_mask;
    v.n_out = m->n_out;
    v.n_in = flip ? m->n_out : m->n_in;
    v.ntiles = (m->n_out + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS;
    v.k3 = m->k3;
    v.flip = flip ? 1 : 0;
    // a submanifold query writes nbr[centre][j] = j (the row itself; flipping maps the
    // centre to itself), so the kernels need not load that column
    v.centre = (m->mode == LAT_SUBM && m->n_in == m->n_out) ? m->k3 / 2 : -1;
    return v;
}

template <typename T>
lat_status launch_conv_simt(const void *x, int cin, const void *w, int cout, const MapView &mv, bool wt, void *y,
                            int32_t *d_status, cudaStream_t s);
template <typename T>
lat_status launch_wgrad_simt(const void *x, int cin, const void *dy, int cout, const lat_kmap *map, float *dw,
                             void *ws, int32_t *d_status, cudaStream_t s);
size_t wgrad_simt_ws_bytes(int cin, int cout, const lat_kmap *map);

bool conv_tc_supported(int kc, int n);
bool wgrad_tc_supported(int cin, int cout);
size_t wgrad_tc_ws_bytes(int cin, int cout, const lat_kmap *map);
lat_status launch_wgrad_tc(bool bf16, const void *x, int cin, const void *dy, int cout, const lat_kmap *map, float *dw,
                           void *ws, int32_t *d_status, cudaStream_t s);
size_t conv_tc_ws_bytes();
lat_status launch_conv_tc(bool bf16, const void *x, int kc, const void *w, int n, int k3, const MapView &mv, bool wt,
                          void *y, void *ws, int32_t *d_status, cudaStream_t s);

}  // namespace lat
