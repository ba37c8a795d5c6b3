// Kernel-map construction / coordinate query (lat_kmap_ws_bytes, lat_kmap_query).
//
// Torch Lattice docs, "Migrating from TorchSparse": kernel-map construction
// and coordinate query are CUDA kernels of the library ("What remains
// familiar", "Sparse tensor expectations"), and the support semantics come
// from the "Convolution mapping" table.  Pipeline (all on `stream`):
//   1. probe:  one thread per output row, K^3 probes of the input table;
//              writes nbr (offset-major, coalesced), mask, and per (offset,
//              block) hit counts from warp ballots.
//   2. scan:   one block turns the counts into pair offsets (offset-major,
//              so pairs come out grouped by offset, rows ascending).
//   3. emit:   re-reads nbr and writes (in, out) pairs at ballot-ranked
//              positions: deterministic, no atomics.
//   4. sort:   stable radix sort of output rows by mask -> perm.
//   5. tiles:  OR of masks over each LAT_TILE_ROWS run of perm -> tile_mask.
#include <cub/device/device_radix_sort.cuh>

#include "common.cuh"

namespace lat {

constexpr int kQueryThreads = 256;
constexpr int kQueryWarps = kQueryThreads / 32;

struct Geom {
    int ks[3], st[3], pd[3];
    int mode;
    int k3;
};

// Input coordinate probed by output row c at offset (ix, iy, iz); false if none.
__device__ __forceinline__ bool query_coord(const Geom &g, const int4 &c, int ix, int iy, int iz, uint64_t &key) {
    int p[3];
    const int q[3] = {c.y, c.z, c.w};
    const int off[3] = {ix, iy, iz};
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        if (g.mode == LAT_TRANSPOSED) {
            const int t = q[a] - off[a] + g.pd[a];
            const int d = floordiv(t, g.st[a]);
            if (d * g.st[a] != t) return false;
            p[a] = d;
        } else {
            p[a] = g.st[a] * q[a] + off[a] - g.pd[a];
        }
    }
    return pack_key(c.x, p[0], p[1], p[2], key);
}

__global__ void __launch_bounds__(kQueryThreads)
kmap_probe_kernel(const Slot *__restrict__ slots, uint64_t cap_mask, const int4 *__restrict__ out_coords,
                  int64_t n_out, int64_t n_in, Geom g, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask,
                  int32_t *__restrict__ iota, int32_t *__restrict__ block_counts, int nblk, int32_t *d_status) {
    __shared__ int s_cnt[32];
    if (threadIdx.x < 32) s_cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const bool live = j < n_out;
    int4 c = make_int4(0, 0, 0, 0);
    if (live) c = __ldg(out_coords + j);
    uint32_t m = 0;
    int32_t bad = 0;
    int k = 0;
    for (int ix = 0; ix < g.ks[0]; ++ix)
        for (int iy = 0; iy < g.ks[1]; ++iy)
            for (int iz = 0; iz < g.ks[2]; ++iz, ++k) {
                int row = -1;
                uint64_t key;
                if (live && query_coord(g, c, ix, iy, iz, key)) row = hash_find(slots, cap_mask, key);
                if (row >= n_in) { bad |= LAT_ERR_BAD_MAP; row = -1; }
                if (live) nbr[int64_t(k) * n_out + j] = row;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, row >= 0);
                if (row >= 0) m |= 1u << k;
                if ((threadIdx.x & 31) == 0 && hits) atomicAdd(&s_cnt[k], __popc(hits));
            }
    if (live) {
        mask[j] = m;
        iota[j] = int32_t(j);
    }
    if (bad) flag(d_status, bad);
    __syncthreads();
    if (threadIdx.x < g.k3) block_counts[int64_t(threadIdx.x) * nblk + blockIdx.x] = s_cnt[threadIdx.x];
}

// Exclusive scan of block_counts (k-major) -> block_offsets; pair_off[k] = start of offset k.
__global__ void __launch_bounds__(1024)
kmap_scan_kernel(const int32_t *__restrict__ block_counts, int64_t *__restrict__ block_offsets, int64_t len,
                 int nblk, int k3, int64_t *__restrict__ pair_off) {
    __shared__ int64_t s_part[1024];
    const int t = threadIdx.x;
    const int64_t per = (len + 1023) / 1024;
    const int64_t lo = min(len, t * per), hi = min(len, lo + per);
    int64_t sum = 0;
    for (int64_t e = lo; e < hi; ++e) sum += block_counts[e];
    s_part[t] = sum;
    __syncthreads();
    for (int d = 1; d < 1024; d <<= 1) {  // Hillis-Steele inclusive scan
        int64_t v = t >= d ? s_part[t - d] : 0;
        __syncthreads();
        s_part[t] += v;
        __syncthreads();
    }
    int64_t run = s_part[t] - sum;
    for (int64_t e = lo; e < hi; ++e) {
        block_offsets[e] = run;
        if (e % nblk == 0) pair_off[e / nblk] = run;
        run += block_counts[e];
    }
    if (t == 1023) pair_off[k3] = s_part[1023];
}

__global__ void __launch_bounds__(kQueryThreads)
kmap_emit_kernel(const int32_t *__restrict__ nbr, int64_t n_out, int k3, const int64_t *__restrict__ block_offsets,
                 int nblk, int32_t *__restrict__ pair_in, int32_t *__restrict__ pair_out, int64_t capacity,
                 int32_t *d_status) {
    __shared__ int s_warp[32][kQueryWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const bool live = j < n_out;
    for (int k = 0; k < k3; ++k) {
        const int row = live ? nbr[int64_t(k) * n_out + j] : -1;
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, row >= 0);
        if (lane == 0) s_warp[k][warp] = __popc(hits);
    }
    __syncthreads();
    bool over = false;
    for (int k = 0; k < k3; ++k) {
        const int row = live ? nbr[int64_t(k) * n_out + j] : -1;
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, row >= 0);
        if (row < 0) continue;
        int64_t pos = block_offsets[int64_t(k) * nblk + blockIdx.x];
        for (int w = 0; w < warp; ++w) pos += s_warp[k][w];
        pos += __popc(hits & ((1u << lane) - 1u));
        if (pos < capacity) {
            pair_in[pos] = row;
            pair_out[pos] = int32_t(j);
        } else {
            over = true;
        }
    }
    if (over) flag(d_status, LAT_ERR_CAPACITY);
}

__global__ void tile_mask_kernel(const uint32_t *__restrict__ sorted_mask, int64_t n, uint32_t *__restrict__ tile_mask,
                                 int64_t ntiles) {
    const int64_t t = blockIdx.x * int64_t(blockDim.x / 32) + (threadIdx.x >> 5);
    if (t >= ntiles) return;
    const int lane = threadIdx.x & 31;
    uint32_t m = 0;
    for (int r = lane; r < LAT_TILE_ROWS; r += 32) {
        const int64_t e = t * LAT_TILE_ROWS + r;
        if (e < n) m |= sorted_mask[e];
    }
    for (int o = 16; o; o >>= 1) m |= __shfl_xor_sync(0xFFFFFFFFu, m, o);
    if (lane == 0) tile_mask[t] = m;
}

struct KmapWs {
    int32_t *block_counts;
    int64_t *block_offsets;
    int32_t *iota;
    uint32_t *sorted_mask;
    void *cub_tmp;
    size_t cub_bytes;
    size_t total;
};

static KmapWs carve_kmap_ws(void *base, int64_t n_out, int k3) {
    KmapWs w{};
    const int nblk = int((n_out + kQueryThreads - 1) / kQueryThreads);
    Carver cv(base);
    w.block_counts = cv.take<int32_t>(size_t(k3) * nblk);
    w.block_offsets = cv.take<int64_t>(size_t(k3) * nblk);
    w.iota = cv.take<int32_t>(size_t(n_out));
    w.sorted_mask = cv.take<uint32_t>(size_t(n_out));
    size_t cub_bytes = 0;
    cub::DeviceRadixSort::SortPairs(nullptr, cub_bytes, (const uint32_t *)nullptr, (uint32_t *)nullptr,
                                    (const int32_t *)nullptr, (int32_t *)nullptr, int(n_out), 0, 32);
    w.cub_bytes = cub_bytes;
    w.cub_tmp = cv.take<char>(cub_bytes);
    w.total = align_up(cv.used, 256);
    return w;
}

bool geom_ok(const lat_geom *g, int &k3) {
    if (!g) return false;
    k3 = 1;
    for (int a = 0; a < 3; ++a) {
        if (g->ksize[a] < 1 || g->stride[a] < 1 || g->pad[a] < 0 || g->pad[a] >= 32768) return false;
        k3 *= g->ksize[a];
    }
    if (k3 > 32) return false;
    if (g->mode == LAT_SUBM) {
        for (int a = 0; a < 3; ++a)
            if (g->stride[a] != 1 || g->ksize[a] % 2 == 0 || g->pad[a] != (g->ksize[a] - 1) / 2) return false;
    } else if (g->mode != LAT_STRIDED && g->mode != LAT_TRANSPOSED) {
        return false;
    }
    return true;
}

}  // namespace lat

extern "C" size_t lat_kmap_ws_bytes(int64_t n_out, int32_t k3) {
    if (n_out < 0 || n_out >= (int64_t(1) << 31) || k3 < 1 || k3 > 32) return 0;
    return lat::carve_kmap_ws(nullptr, n_out, k3).total;
}

extern "C" lat_status lat_kmap_query(const void *table, size_t table_bytes, const int32_t *out_coords,
                                     const lat_geom *geom, lat_kmap *map, void *ws, size_t ws_bytes,
                                     int32_t *d_status, lat_stream stream) {
    using namespace lat;
    int k3 = 0;
    if (!map || !geom_ok(geom, k3) || map->k3 != k3) return LAT_ERR_ARG;
    const int64_t n_out = map->n_out, n_in = map->n_in;
    if (n_out < 0 || n_out >= (int64_t(1) << 31) || n_in < 0 || n_in >= (int64_t(1) << 31)) return LAT_ERR_ARG;
    if (!table || table_bytes % sizeof(Slot) || !pow2(table_bytes / sizeof(Slot))) return LAT_ERR_ARG;
    if (map->pair_capacity < 0 || !map->pair_off) return LAT_ERR_ARG;
    if (n_out > 0 && (!out_coords || !map->nbr || !map->mask || !map->perm || !map->tile_mask)) return LAT_ERR_ARG;
    if (map->pair_capacity > 0 && (!map->pair_in || !map->pair_out)) return LAT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(out_coords) % 16 || reinterpret_cast<uintptr_t>(table) % 16) return LAT_ERR_ARG;
    const KmapWs need = carve_kmap_ws(nullptr, n_out, k3);
    if (ws_bytes < need.total || (need.total && !ws)) return LAT_ERR_WORKSPACE;
    map->mode = geom->mode;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (n_out == 0) {
        LAT_CUDA_TRY(cudaMemsetAsync(map->pair_off, 0, sizeof(int64_t) * (k3 + 1), s));
        return LAT_OK;
    }
    KmapWs w = carve_kmap_ws(ws, n_out, k3);
    Geom g{};
    for (int a = 0; a < 3; ++a) {
        g.ks[a] = geom->ksize[a];
        g.st[a] = geom->stride[a];
        g.pd[a] = geom->pad[a];
    }
    g.mode = geom->mode;
    g.k3 = k3;
    const int nblk = int((n_out + kQueryThreads - 1) / kQueryThreads);
    const uint64_t cap_mask = table_bytes / sizeof(Slot) - 1;
    kmap_probe_kernel<<<nblk, kQueryThreads, 0, s>>>(static_cast<const Slot *>(table), cap_mask,
                                                      reinterpret_cast<const int4 *>(out_coords), n_out, n_in, g,
                                                      map->nbr, map->mask, w.iota, w.block_counts, nblk, d_status);
    LAT_CUDA_TRY(cudaGetLastError());
    kmap_scan_kernel<<<1, 1024, 0, s>>>(w.block_counts, w.block_offsets, int64_t(k3) * nblk, nblk, k3, map->pair_off);
    LAT_CUDA_TRY(cudaGetLastError());
    kmap_emit_kernel<<<nblk, kQueryThreads, 0, s>>>(map->nbr, n_out, k3, w.block_offsets, nblk, map->pair_in,
                                                     map->pair_out, map->pair_capacity, d_status);
    LAT_CUDA_TRY(cudaGetLastError());
    size_t cub_bytes = w.cub_bytes;
    LAT_CUDA_TRY(cub::DeviceRadixSort::SortPairs(w.cub_tmp, cub_bytes, map->mask, w.sorted_mask, w.iota, map->perm,
                                                 int(n_out), 0, k3, s));
    const int64_t ntiles = (n_out + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS;
    tile_mask_kernel<<<unsigned((ntiles + 7) / 8), 256, 0, s>>>(w.sorted_mask, n_out, map->tile_mask, ntiles);
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}
