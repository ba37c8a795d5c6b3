// Sparse pooling over a kernel map and dense materialization
// (lat_sparse_pool, lat_to_dense).
//
// Torch Lattice docs, "Migrating from TorchSparse", "What remains familiar":
// pooling and dense conversion are among the library's CUDA kernels.  The
// pages fix no formula; the plainest reading is taken:
//   pool:  y[j][c] = max (or mean) over the offsets k with a neighbour of
//          x[nbr[k][j]][c]; rows with no neighbour get 0.  fp32 arithmetic,
//          the mean is the sum in offset order divided by the neighbour count,
//          one rounding to the output type.
//   dense: a channels-last grid over a caller-given box, zero where no row
//          lies; every row inside the box writes its features to its cell.
// Both are memory-bound gathers / scatters on CUDA cores: one thread per (row,
// 8-channel group) -- a 2D block, so no thread divides its index -- with
// 16-byte (fp16/bf16) or 2 x 16-byte (fp32) accesses.
#include "common.cuh"

namespace lat {

template <typename T>
__device__ __forceinline__ void st8(T *p, const float (&v)[8]) {
    if constexpr (sizeof(T) == 4) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        uint4 o;
        T *e = reinterpret_cast<T *>(&o);
#pragma unroll
        for (int c = 0; c < 8; ++c) e[c] = Elem<T>::from_f(v[c]);
        *reinterpret_cast<uint4 *>(p) = o;
    }
}

// Raw 16-byte (fp16/bf16) or 32-byte (fp32) slice of one row: 8 channels.
template <typename T> struct Slice {
    uint4 v[sizeof(T) / 2];
};

template <typename T>
__device__ __forceinline__ void ld_slice(const T *p, Slice<T> &s) {
#pragma unroll
    for (int h = 0; h < int(sizeof(T) / 2); ++h) s.v[h] = __ldg(reinterpret_cast<const uint4 *>(p) + h);
}

template <typename T>
__device__ __forceinline__ void unpack(const Slice<T> &s, float (&v)[8]) {
    const T *e = reinterpret_cast<const T *>(s.v);
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = Elem<T>::to_f(e[c]);
}

// One thread per (output row, group of 8 channels); the offsets come from the row's mask.
// The next neighbour's row index is loaded while the current neighbour's features are in
// flight, so a row with m neighbours costs m + 2 dependent memory round trips, not 2m + 1.
// (Wider batches of loads per thread measured slower here: the extra registers cost more
// occupancy than the extra loads in flight gain, since most rows have one to four
// neighbours.)
template <typename T, bool MAX>
__global__ void __launch_bounds__(256)
pool_kernel(const T *__restrict__ x, int c, const int32_t *__restrict__ nbr, const uint32_t *__restrict__ mask,
            int k3, int64_t n_in, int64_t n_out, T *__restrict__ y, int32_t *d_status) {
    pdl_enter();
    // threadIdx.x = 8-channel group, threadIdx.y = row of the block
    const int64_t j = blockIdx.x * int64_t(blockDim.y) + threadIdx.y;
    if (j >= n_out) return;
    const int cg = threadIdx.x;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = MAX ? -INFINITY : 0.f;
    int cnt = 0;
    int32_t bad = 0;
    const uint32_t valid = k3 >= 32 ? ~0u : (1u << k3) - 1u;
    const uint32_t mj = __ldg(mask + j);
    if (mj & ~valid) bad |= LAT_ERR_BAD_MAP;
    uint32_t m = mj & valid;
    const T *xs = x + cg * 8;
    int i = 0;
    bool have = m != 0;
    if (have) {
        i = __ldg(nbr + int64_t(__ffs(m) - 1) * n_out + j);
        m &= m - 1;
    }
    while (have) {
        const bool more = m != 0;
        int i_next = 0;
        if (more) {
            i_next = __ldg(nbr + int64_t(__ffs(m) - 1) * n_out + j);
            m &= m - 1;
        }
        if (i >= 0 && i < n_in) {
            Slice<T> row;
            ld_slice<T>(xs + int64_t(i) * c, row);
            float v[8];
            unpack<T>(row, v);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = MAX ? fmaxf(acc[e], v[e]) : acc[e] + v[e];
            ++cnt;
        } else {
            bad |= LAT_ERR_BAD_MAP;
        }
        i = i_next;
        have = more;
    }
    if (bad) flag(d_status, bad);
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = cnt == 0 ? 0.f : (MAX ? acc[e] : acc[e] / float(cnt));
    st8<T>(y + j * c + cg * 8, out);
}

struct Box {
    int ox, oy, oz, sx, sy, sz, batch;
};

// Scatter every row inside the box into its cell of the zeroed channels-last grid.
template <typename T>
__global__ void __launch_bounds__(256)
dense_scatter_kernel(const int4 *__restrict__ coords, int64_t n, const T *__restrict__ feats, int c, Box bx,
                     T *__restrict__ out, int32_t *d_status) {
    pdl_enter();
    const int64_t i = blockIdx.x * int64_t(blockDim.y) + threadIdx.y;
    if (i >= n) return;
    const int cg = threadIdx.x;
    const int4 q = __ldg(coords + i);
    const int x = q.y - bx.ox, y = q.z - bx.oy, z = q.w - bx.oz;
    if (q.x < 0 || q.x >= bx.batch || x < 0 || x >= bx.sx || y < 0 || y >= bx.sy || z < 0 || z >= bx.sz) {
        if (cg == 0) flag(d_status, LAT_ERR_COORD_RANGE);
        return;
    }
    const int64_t cell = ((int64_t(q.x) * bx.sx + x) * bx.sy + y) * bx.sz + z;
    Slice<T> v;
    ld_slice<T>(feats + i * c + cg * 8, v);
#pragma unroll
    for (int h = 0; h < int(sizeof(T) / 2); ++h) reinterpret_cast<uint4 *>(out + cell * c + cg * 8)[h] = v.v[h];
}

// Thread block of the pooling / dense kernels: x = the row's 8-channel groups
// (c / 8 <= 256), y = rows, about 256 threads.
static dim3 rows_block(int c) {
    const int groups = c / 8;
    return dim3(unsigned(groups), unsigned(groups >= 256 ? 1 : 256 / groups));
}

template <typename T>
static lat_status launch_pool(const void *x, int c, const lat_kmap *map, int op, void *y, int32_t *d_status,
                              cudaStream_t s) {
    if (map->n_out == 0) return LAT_OK;
    const dim3 block = rows_block(c);
    const dim3 blocks(unsigned((map->n_out + block.y - 1) / block.y));
    if (op == LAT_POOL_MAX)
        LAT_CUDA_TRY(launch_pdl(pool_kernel<T, true>, blocks, block, 0, s, static_cast<const T *>(x), c,
                                map->nbr, map->mask, map->k3, map->n_in, map->n_out, static_cast<T *>(y), d_status));
    else
        LAT_CUDA_TRY(launch_pdl(pool_kernel<T, false>, blocks, block, 0, s, static_cast<const T *>(x), c,
                                map->nbr, map->mask, map->k3, map->n_in, map->n_out, static_cast<T *>(y), d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

template <typename T>
static lat_status launch_dense(const int32_t *coords, int64_t n, const void *feats, int c, const Box &bx, void *out,
                               int32_t *d_status, cudaStream_t s) {
    const size_t cells = size_t(bx.batch) * bx.sx * bx.sy * bx.sz;
    LAT_CUDA_TRY(cudaMemsetAsync(out, 0, cells * c * sizeof(T), s));
    if (n == 0) return LAT_OK;
    const dim3 block = rows_block(c);
    LAT_CUDA_TRY(launch_pdl(dense_scatter_kernel<T>, dim3(unsigned((n + block.y - 1) / block.y)), block, 0, s,
                            reinterpret_cast<const int4 *>(coords), n, static_cast<const T *>(feats), c, bx,
                            static_cast<T *>(out), d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

static bool aligned16(const void *p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

}  // namespace lat

extern "C" lat_status lat_sparse_pool(const void *x, int32_t c, const lat_kmap *map, int32_t op, void *y,
                                      lat_dtype dtype, int32_t *d_status, lat_stream stream) {
    using namespace lat;
    if (!map || map->k3 < 1 || map->k3 > 32 || map->n_in < 0 || map->n_out < 0) return LAT_ERR_ARG;
    if (map->n_out >= (int64_t(1) << 31) || map->n_in >= (int64_t(1) << 31)) return LAT_ERR_ARG;
    if (c < 8 || c % 8 || c > 2048 || (op != LAT_POOL_MAX && op != LAT_POOL_AVG)) return LAT_ERR_ARG;
    if (map->n_out > 0 && (!map->nbr || !map->mask || !y || (map->n_in > 0 && !x))) return LAT_ERR_ARG;
    if (!aligned16(x) || !aligned16(y)) return LAT_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (dtype) {
        case LAT_F32: return launch_pool<float>(x, c, map, op, y, d_status, s);
        case LAT_F16: return launch_pool<__half>(x, c, map, op, y, d_status, s);
        case LAT_BF16: return launch_pool<__nv_bfloat16>(x, c, map, op, y, d_status, s);
    }
    return LAT_ERR_ARG;
}

extern "C" lat_status lat_to_dense(const int32_t *coords, int64_t n, const void *feats, int32_t c, lat_dtype dtype,
                                   const int32_t *origin, const int32_t *shape, int32_t batch, void *out,
                                   int32_t *d_status, lat_stream stream) {
    using namespace lat;
    if (n < 0 || n >= (int64_t(1) << 31) || c < 8 || c % 8 || c > 2048 || !origin || !shape || batch < 1 || !out)
        return LAT_ERR_ARG;
    if (n > 0 && (!coords || !feats)) return LAT_ERR_ARG;
    for (int a = 0; a < 3; ++a)
        if (shape[a] < 1) return LAT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(coords) % 16 || !aligned16(feats) || !aligned16(out)) return LAT_ERR_ARG;
    const Box bx{origin[0], origin[1], origin[2], shape[0], shape[1], shape[2], batch};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (dtype) {
        case LAT_F32: return launch_dense<float>(coords, n, feats, c, bx, out, d_status, s);
        case LAT_F16: return launch_dense<__half>(coords, n, feats, c, bx, out, d_status, s);
        case LAT_BF16: return launch_dense<__nv_bfloat16>(coords, n, feats, c, bx, out, d_status, s);
    }
    return LAT_ERR_ARG;
}
