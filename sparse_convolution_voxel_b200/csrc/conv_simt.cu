// CUDA-core sparse convolution (fp32 path; FFMA, no TF32).
//
// Output-stationary implicit GEMM over the kernel map: every output row is
// owned by one thread group, accumulates sum_k x[nbr[k][j]] . W[k] in fp32
// registers over the offsets its tile touches, and is written once -- no
// atomics (TorchSparse++ abstract: implicit GEMM overlaps computation with
// memory access; migration page, "Backend and configuration differences":
// every dataflow gives the same result for a fixed relation and weights).
//
// Tiles are LAT_TILE_ROWS consecutive entries of the mask-sorted row order
// `perm`, and only offsets in the tile's mask union are visited.  The same
// kernel computes the data gradient with W[k]^T and, for a submanifold map,
// the flipped offset (the pair (i, j, k) sits at nbr[k3-1-k][i]).
//
// Weight gradient: pairs of each offset are cut into fixed chunks; one block
// reduces a chunk into an fp32 partial, then the partials of each offset are
// summed in chunk order, so the result is deterministic.
#include "common.cuh"
#include "conv_common.cuh"

namespace lat {

constexpr int kSimtThreads = 256;
constexpr int kCoGroup = 8;  // output channels per thread item

template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__half>(const __half *p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const __half2 *h = reinterpret_cast<const __half2 *>(&a);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
    }
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&a);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
    }
}

template <typename T>
__device__ __forceinline__ void store8(T *p, const float (&v)[8]) {
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

// One tile = LAT_TILE_ROWS rows of perm.  Items (row r, channel group g) are laid
// out g-major so that a warp holds 32 rows of one channel group: its weight reads
// are warp-uniform (broadcast) and its feature reads are one row per lane.
// WT: the weight used at offset k is W[k]^T (data gradient).
template <typename T, bool WT>
__global__ void __launch_bounds__(kSimtThreads)
conv_simt_kernel(const T *__restrict__ x, int cin, const T *__restrict__ w, int cout, MapView mv,
                 T *__restrict__ y, int32_t *d_status) {
    const int ngroups = cout / kCoGroup;
    const int items = LAT_TILE_ROWS * ngroups;
    // weight element (ci, co) of the GEMM at offset k
    const int64_t wk_stride = int64_t(cin) * cout;
    int32_t bad = 0;
    for (int64_t t = blockIdx.x; t < mv.ntiles; t += gridDim.x) {
        const uint32_t tmask = mv.tile_mask_at(t);
        const int64_t row0 = t * LAT_TILE_ROWS;
        for (int it = threadIdx.x; it < items; it += kSimtThreads) {
            const int r = it % LAT_TILE_ROWS, g = it / LAT_TILE_ROWS;
            if (row0 + r >= mv.n_out) continue;
            const int j = mv.perm[row0 + r];
            float acc[kCoGroup];
#pragma unroll
            for (int c = 0; c < kCoGroup; ++c) acc[c] = 0.f;
            for (uint32_t m = tmask; m; m &= m - 1) {
                const int k = __ffs(m) - 1;
                const int src = mv.neighbour(k, j);
                if (src < 0) continue;
                if (src >= mv.n_in) { bad |= LAT_ERR_BAD_MAP; continue; }
                const T *xr = x + int64_t(src) * cin;
                const T *wk = w + int64_t(k) * wk_stride;
                for (int c0 = 0; c0 < cin; c0 += 8) {
                    float xv[8];
                    load8<T>(xr + c0, xv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int ci = c0 + e;
                        float wv[8];
                        if constexpr (!WT) {
                            load8<T>(wk + int64_t(ci) * cout + g * kCoGroup, wv);
                        } else {  // W^T: element (ci, co) = W[k][co][ci], W[k] is (cout x cin) here
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                wv[c] = Elem<T>::to_f(wk[int64_t(g * kCoGroup + c) * cin + ci]);
                        }
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc[c] = fmaf(xv[e], wv[c], acc[c]);
                    }
                }
            }
            store8<T>(y + int64_t(j) * cout + g * kCoGroup, acc);
        }
    }
    if (bad) flag(d_status, bad);
}

// Work units of the weight gradient: fixed chunks of kWgradChunk pairs inside one offset.
__global__ void wgrad_units_kernel(const int64_t *__restrict__ pair_off, int k3, int64_t capacity, int chunk,
                                   int32_t *__restrict__ unit_base) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int32_t u = 0;
    for (int k = 0; k < k3; ++k) {
        unit_base[k] = u;
        const int64_t lo = min(pair_off[k], capacity), hi = min(pair_off[k + 1], capacity);
        u += int32_t((hi - lo + chunk - 1) / chunk);
    }
    unit_base[k3] = u;
}

constexpr int kWgradBatch = 32;

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
wgrad_simt_kernel(const T *__restrict__ x, int cin, const T *__restrict__ dy, int cout, const int64_t *__restrict__ pair_off,
                  const int32_t *__restrict__ pair_in, const int32_t *__restrict__ pair_out, int64_t capacity, int k3,
                  int64_t n_in, int64_t n_out, const int32_t *__restrict__ unit_base, int chunk, float *__restrict__ partial,
                  int32_t *d_status) {
    extern __shared__ float smem[];
    float *xs = smem;                       // [kWgradBatch][cin]
    float *gs = smem + kWgradBatch * cin;   // [kWgradBatch][cout]
    const int nelem = cin * cout;
    const int32_t units = unit_base[k3];
    int32_t bad = 0;
    for (int32_t u = blockIdx.x; u < units; u += gridDim.x) {
        int k = 0;
        while (unit_base[k + 1] <= u) ++k;
        const int64_t lo = min(pair_off[k], capacity) + int64_t(u - unit_base[k]) * chunk;
        const int64_t hi = min(lo + chunk, min(pair_off[k + 1], capacity));
        float acc[64];  // up to 256*256/256 elements per thread would not fit; cap nelem/threads at 64
        const int per = (nelem + kSimtThreads - 1) / kSimtThreads;
#pragma unroll
        for (int e = 0; e < 64; ++e) acc[e] = 0.f;
        for (int64_t p0 = lo; p0 < hi; p0 += kWgradBatch) {
            const int np = int(hi - p0 < kWgradBatch ? hi - p0 : int64_t(kWgradBatch));
            __syncthreads();
            for (int idx = threadIdx.x; idx < kWgradBatch * (cin + cout); idx += kSimtThreads) {
                const int p = idx / (cin + cout), c = idx % (cin + cout);
                float v = 0.f;
                if (p < np) {
                    if (c < cin) {
                        const int i = pair_in[p0 + p];
                        if (i >= 0 && i < n_in) v = Elem<T>::to_f(x[int64_t(i) * cin + c]);
                        else bad |= LAT_ERR_BAD_MAP;
                    } else {
                        const int j = pair_out[p0 + p];
                        if (j >= 0 && j < n_out) v = Elem<T>::to_f(dy[int64_t(j) * cout + (c - cin)]);
                        else bad |= LAT_ERR_BAD_MAP;
                    }
                }
                if (c < cin) xs[p * cin + c] = v; else gs[p * cout + (c - cin)] = v;
            }
            __syncthreads();
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                if (e >= per) break;
                const int el = threadIdx.x + e * kSimtThreads;
                if (el >= nelem) break;
                const int ci = el / cout, co = el % cout;
                float a = acc[e];
                for (int p = 0; p < np; ++p) a = fmaf(xs[p * cin + ci], gs[p * cout + co], a);
                acc[e] = a;
            }
        }
        float *dst = partial + int64_t(u) * nelem;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
            if (e >= per) break;
            const int el = threadIdx.x + e * kSimtThreads;
            if (el < nelem) dst[el] = acc[e];
        }
        __syncthreads();
    }
    if (bad) flag(d_status, bad);
}

__global__ void wgrad_reduce_kernel(const float *__restrict__ partial, const int32_t *__restrict__ unit_base, int k3,
                                    int nelem, float *__restrict__ dw) {
    const int k = blockIdx.y;
    const int el = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= k3 || el >= nelem) return;
    float s = 0.f;
    for (int32_t u = unit_base[k]; u < unit_base[k + 1]; ++u) s += partial[int64_t(u) * nelem + el];
    dw[int64_t(k) * nelem + el] = s;
}

// ----------------------------------------------------------------------------- host side
constexpr int kWgradChunkSimt = 1024;

size_t wgrad_simt_ws_bytes(int cin, int cout, const lat_kmap *map) {
    const int64_t units = (map->pair_capacity + kWgradChunkSimt - 1) / kWgradChunkSimt + map->k3;
    Carver cv(nullptr);
    cv.take<int32_t>(size_t(map->k3) + 1);
    cv.take<float>(size_t(units) * cin * cout);
    return align_up(cv.used, 256);
}

template <typename T>
lat_status launch_conv_simt(const void *x, int cin, const void *w, int cout, const MapView &mv, bool wt, void *y,
                            int32_t *d_status, cudaStream_t s) {
    if (mv.ntiles == 0) return LAT_OK;
    const int64_t grid = std::min<int64_t>(mv.ntiles, int64_t(num_sms()) * 8);
    if (wt)
        conv_simt_kernel<T, true><<<unsigned(grid), kSimtThreads, 0, s>>>(
            static_cast<const T *>(x), cin, static_cast<const T *>(w), cout, mv, static_cast<T *>(y), d_status);
    else
        conv_simt_kernel<T, false><<<unsigned(grid), kSimtThreads, 0, s>>>(
            static_cast<const T *>(x), cin, static_cast<const T *>(w), cout, mv, static_cast<T *>(y), d_status);
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

template lat_status launch_conv_simt<float>(const void *, int, const void *, int, const MapView &, bool, void *,
                                            int32_t *, cudaStream_t);
template lat_status launch_conv_simt<__half>(const void *, int, const void *, int, const MapView &, bool, void *,
                                             int32_t *, cudaStream_t);
template lat_status launch_conv_simt<__nv_bfloat16>(const void *, int, const void *, int, const MapView &, bool,
                                                    void *, int32_t *, cudaStream_t);

template <typename T>
lat_status launch_wgrad_simt(const void *x, int cin, const void *dy, int cout, const lat_kmap *map, float *dw,
                             void *ws, int32_t *d_status, cudaStream_t s) {
    if (cin * cout > 64 * kSimtThreads) return LAT_ERR_UNSUPPORTED;
    const int64_t units_max = (map->pair_capacity + kWgradChunkSimt - 1) / kWgradChunkSimt + map->k3;
    Carver cv(ws);
    int32_t *unit_base = cv.take<int32_t>(size_t(map->k3) + 1);
    float *partial = cv.take<float>(size_t(units_max) * cin * cout);
    wgrad_units_kernel<<<1, 32, 0, s>>>(map->pair_off, map->k3, map->pair_capacity, kWgradChunkSimt, unit_base);
    LAT_CUDA_TRY(cudaGetLastError());
    const size_t smem = sizeof(float) * kWgradBatch * (cin + cout);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(units_max, int64_t(num_sms()) * 4));
    wgrad_simt_kernel<T><<<unsigned(grid), kSimtThreads, smem, s>>>(
        static_cast<const T *>(x), cin, static_cast<const T *>(dy), cout, map->pair_off, map->pair_in, map->pair_out,
        map->pair_capacity, map->k3, map->n_in, map->n_out, unit_base, kWgradChunkSimt, partial, d_status);
    LAT_CUDA_TRY(cudaGetLastError());
    const int nelem = cin * cout;
    dim3 rg((nelem + 255) / 256, map->k3);
    wgrad_reduce_kernel<<<rg, 256, 0, s>>>(partial, unit_base, map->k3, nelem, dw);
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

template lat_status launch_wgrad_simt<float>(const void *, int, const void *, int, const lat_kmap *, float *, void *,
                                             int32_t *, cudaStream_t);
template lat_status launch_wgrad_simt<__half>(const void *, int, const void *, int, const lat_kmap *, float *, void *,
                                              int32_t *, cudaStream_t);
template lat_status launch_wgrad_simt<__nv_bfloat16>(const void *, int, const void *, int, const lat_kmap *, float *,
                                                     void *, int32_t *, cudaStream_t);

}  // namespace lat
