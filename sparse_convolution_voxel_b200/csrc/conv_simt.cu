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

// One block per tile of LAT_TILE_ROWS rows of perm, one thread per row.  For
// every 32 output channels, each offset of the tile's mask union stages the
// matching W[k] slice (Cin x 32, fp32) in shared memory; every thread whose row
// has that neighbour reads its input row (8 channels per vector load) and does
// 32 FMAs per input channel against warp-uniform (broadcast) weight reads.
// WT: the weight used at offset k is W[k]^T (data gradient).
constexpr int kCoChunk = 32;

template <typename T, bool WT>
__global__ void __launch_bounds__(LAT_TILE_ROWS)
conv_simt_kernel(const T *__restrict__ x, int cin, const T *__restrict__ w, int cout, MapView mv,
                 T *__restrict__ y, int32_t *d_status) {
    pdl_enter();
    extern __shared__ float s_w[];  // [cin][kCoChunk]
    const int64_t t = blockIdx.x;
    const uint32_t tmask = mv.tile_mask_at(t);
    const int64_t row = t * LAT_TILE_ROWS + threadIdx.x;
    const int j = row < mv.n_out ? mv.perm[row] : -1;
    const int64_t wk_stride = int64_t(cin) * cout;
    int32_t bad = 0;
    for (int co0 = 0; co0 < cout; co0 += kCoChunk) {
        const int cw = min(kCoChunk, cout - co0);
        float acc[kCoChunk];
#pragma unroll
        for (int c = 0; c < kCoChunk; ++c) acc[c] = 0.f;
        for (uint32_t m = tmask; m; m &= m - 1) {
            const int k = __ffs(m) - 1;
            int src = j >= 0 ? mv.neighbour(k, j) : -1;
            if (src >= mv.n_in) {
                bad |= LAT_ERR_BAD_MAP;
                src = -1;
            }
            const T *wk = w + int64_t(k) * wk_stride;
            __syncthreads();
            for (int e = threadIdx.x; e < cin * kCoChunk; e += LAT_TILE_ROWS) {
                const int ci = e / kCoChunk, c = e % kCoChunk;
                float v = 0.f;
                if (c < cw) {
                    // (ci, co) of the GEMM: W[k][ci][co], or W[k][co][ci] for W^T
                    v = WT ? Elem<T>::to_f(wk[int64_t(co0 + c) * cin + ci])
                           : Elem<T>::to_f(wk[int64_t(ci) * cout + co0 + c]);
                }
                s_w[e] = v;
            }
            __syncthreads();
            if (src < 0) continue;
            const T *xr = x + int64_t(src) * cin;
            for (int c0 = 0; c0 < cin; c0 += 8) {
                float xv[8];
                load8<T>(xr + c0, xv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 *wr = reinterpret_cast<const float4 *>(s_w + (c0 + e) * kCoChunk);
#pragma unroll
                    for (int q = 0; q < kCoChunk / 4; ++q) {
                        if (4 * q >= cw) break;  // block-uniform: narrow outputs skip the unused columns
                        const float4 wv = wr[q];
                        acc[4 * q] = fmaf(xv[e], wv.x, acc[4 * q]);
                        acc[4 * q + 1] = fmaf(xv[e], wv.y, acc[4 * q + 1]);
                        acc[4 * q + 2] = fmaf(xv[e], wv.z, acc[4 * q + 2]);
                        acc[4 * q + 3] = fmaf(xv[e], wv.w, acc[4 * q + 3]);
                    }
                }
            }
        }
        if (j >= 0) {
            T *yr = y + int64_t(j) * cout + co0;
#pragma unroll
            for (int g = 0; g < kCoChunk / 8; ++g) {
                if (g * 8 < cw) {
                    float v[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) v[c] = acc[g * 8 + c];
                    store8<T>(yr + g * 8, v);
                }
            }
        }
    }
    if (bad) flag(d_status, bad);
}

// Small problems (too few 128-row tiles to fill the GPU): one warp per output
// row, lane k takes offset k, so a row's offsets are gathered in parallel
// instead of one after another.  The block stages W transposed as
// s_w[ci][co][k] (lanes read consecutive words: no bank conflicts); each lane
// forms x[nbr[k][j]] . W[k] for the row's cout outputs and the warp sums the
// offsets with a fixed xor-butterfly (deterministic).  Needs k3 <= 32,
// cout <= 32 and cin * cout * 32 floats of shared memory.
constexpr int kRowsPerBlock = 8;

template <typename T, bool WT>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
conv_rows_kernel(const T *__restrict__ x, int cin, const T *__restrict__ w, int cout, MapView mv,
                 T *__restrict__ y, int32_t *d_status) {
    pdl_enter();
    extern __shared__ float s_w[];  // [cin][cout][32]
    const int lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < cin * cout * 32; e += blockDim.x) {
        const int k = e & 31, co = (e >> 5) % cout, ci = (e >> 5) / cout;
        float v = 0.f;
        if (k < mv.k3) {
            // (ci, co) of the GEMM: W[k][ci][co], or W[k][co][ci] for W^T
            const T *wk = w + int64_t(k) * cin * cout;
            v = WT ? Elem<T>::to_f(wk[int64_t(co) * cin + ci]) : Elem<T>::to_f(wk[int64_t(ci) * cout + co]);
        }
        s_w[e] = v;
    }
    __syncthreads();
    const int64_t j = blockIdx.x * int64_t(kRowsPerBlock) + (threadIdx.x >> 5);
    if (j >= mv.n_out) return;
    int32_t bad = 0;
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = 0.f;
    int src = lane < mv.k3 ? mv.neighbour(lane, j) : -1;
    if (src >= mv.n_in) {
        bad |= LAT_ERR_BAD_MAP;
        src = -1;
    }
    if (src >= 0) {
        const T *xr = x + int64_t(src) * cin;
        for (int c0 = 0; c0 < cin; c0 += 8) {
            float xv[8];
            load8<T>(xr + c0, xv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float *wr = s_w + ((c0 + e) * cout) * 32 + lane;
#pragma unroll
                for (int co = 0; co < 32; ++co)
                    if (co < cout) acc[co] = fmaf(xv[e], wr[co * 32], acc[co]);
            }
        }
    }
#pragma unroll
    for (int co = 0; co < 32; ++co) {
        if (co >= cout) break;
#pragma unroll
        for (int o = 16; o; o >>= 1) acc[co] += __shfl_xor_sync(0xFFFFFFFFu, acc[co], o);
    }
    // lane co writes output channel co (every lane holds every total)
    float mine = 0.f;
#pragma unroll
    for (int co = 0; co < 32; ++co)
        if (co == lane) mine = acc[co];
    if (lane < cout) y[j * cout + lane] = Elem<T>::from_f(mine);
    if (bad) flag(d_status, bad);
}

// Work units of the weight gradient: fixed chunks of kWgradChunk pairs inside one offset.
// First unit of every offset and the total (unit_base[k3]); one warp, lane k
// handles offset k (k3 <= 32): offset k's clamped pairs make ceil(P_k / chunk) units.
__global__ void wgrad_units_kernel(const int64_t *__restrict__ pair_off, int k3, int64_t capacity, int chunk,
                                   int32_t *__restrict__ unit_base) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t P = min(pair_off[k3], capacity);
    const int64_t lo = lane < k3 ? min(pair_off[lane], capacity) : P;
    const int64_t up = __shfl_down_sync(0xFFFFFFFFu, lo, 1);
    const int64_t hi = lane == 31 ? P : up;
    const int32_t units = lane < k3 ? int32_t((hi - lo + chunk - 1) / chunk) : 0;
    int32_t incl = units;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
    }
    if (lane < k3) unit_base[lane] = incl - units;
    if (lane == 31) unit_base[k3] = incl;
}

// One block of 8 warps per (unit, group of slices).  A slice is 256 consecutive
// elements of the Cin x Cout partial: lane l owns 8 consecutive output channels
// of one input channel, so for every pair all 32 lanes read the same x row (one
// value each) and the same dy row (one 32-byte piece each) -- coalesced,
// broadcast loads -- and do 8 FMAs.  With nslices >= 8 each warp takes one
// slice over the unit's pairs; with fewer (small Cin x Cout) the warps of a
// slice split the pairs into parts and add their sums in shared memory in part
// order.  Pair order and part order are fixed, so each partial is deterministic.
constexpr int kWgradSlice = 256;
constexpr int kWgradWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kWgradWarps * 32)
wgrad_simt_kernel(const T *__restrict__ x, int cin, const T *__restrict__ dy, int cout, const int64_t *__restrict__ pair_off,
                  const int32_t *__restrict__ pair_in, const int32_t *__restrict__ pair_out, int64_t capacity, int k3,
                  int64_t n_in, int64_t n_out, const int32_t *__restrict__ unit_base, int chunk, float *__restrict__ partial,
                  int32_t *d_status) {
    pdl_enter();
    __shared__ float s_part[kWgradWarps][kWgradSlice];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nelem = cin * cout;
    const int nslices = (nelem + kWgradSlice - 1) / kWgradSlice;
    // warps per slice (parts of the pair range) and slices per block
    const int parts = nslices >= kWgradWarps ? 1 : (kWgradWarps % nslices == 0 ? kWgradWarps / nslices : 1);
    const int per_block = kWgradWarps / parts;
    const int groups = (nslices + per_block - 1) / per_block;
    const int32_t u = int32_t(blockIdx.x / groups);
    const int slice = int(blockIdx.x % groups) * per_block + warp / parts;
    const int part = warp % parts;
    const bool unit_ok = u < unit_base[k3];
    const int e0 = slice * kWgradSlice + lane * 8;
    const bool own = unit_ok && slice < nslices && e0 < nelem;
    const int ci = own ? e0 / cout : 0, co0 = own ? e0 % cout : 0;
    int64_t lo = 0, hi = 0;
    if (unit_ok) {
        int k = 0;
        while (unit_base[k + 1] <= u) ++k;
        const int64_t ulo = min(pair_off[k], capacity) + int64_t(u - unit_base[k]) * chunk;
        const int64_t uhi = min(ulo + chunk, min(pair_off[k + 1], capacity));
        const int64_t per = (uhi - ulo + parts - 1) / parts;
        lo = min(uhi, ulo + per * part);
        hi = min(uhi, lo + per);
    }
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    int32_t bad = 0;
    if (own) {
        for (int64_t p0 = lo; p0 < hi; p0 += 4) {
            float xv[4], gv[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t p = p0 + q;
                int i = -1, jj = -1;
                if (p < hi) {
                    i = __ldg(pair_in + p);
                    jj = __ldg(pair_out + p);
                    if (i < 0 || i >= n_in || jj < 0 || jj >= n_out) {
                        bad |= LAT_ERR_BAD_MAP;
                        i = jj = -1;
                    }
                }
                xv[q] = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) gv[q][c] = 0.f;
                if (i >= 0) {
                    xv[q] = Elem<T>::to_f(x[int64_t(i) * cin + ci]);
                    load8<T>(dy + int64_t(jj) * cout + co0, gv[q]);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = fmaf(xv[q], gv[q][c], acc[c]);
        }
    }
    if (parts > 1) {
#pragma unroll
        for (int c = 0; c < 8; ++c) s_part[warp][lane * 8 + c] = acc[c];
        __syncthreads();
        if (part == 0 && own) {
            for (int q = 1; q < parts; ++q)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] += s_part[warp + q][lane * 8 + c];
        }
    }
    if (own && part == 0) {
        float *dst = partial + int64_t(u) * nelem + e0;
        reinterpret_cast<float4 *>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        reinterpret_cast<float4 *>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    if (bad) flag(d_status, bad);
}

__global__ void wgrad_reduce_kernel(const float *__restrict__ partial, const int32_t *__restrict__ unit_base, int k3,
                                    int nelem, float *__restrict__ dw) {
    pdl_enter();
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
    if (mv.ntiles >= (int64_t(1) << 31)) return LAT_ERR_UNSUPPORTED;
    // too few tiles to fill the GPU: one warp per row, offsets across the lanes
    const size_t rows_smem = sizeof(float) * size_t(cin) * size_t(cout) * 32;
    if (mv.ntiles < 2 * int64_t(num_sms()) && mv.k3 <= 32 && cout <= 32 && rows_smem <= 96 * 1024) {
        const dim3 grid(unsigned((mv.n_out + kRowsPerBlock - 1) / kRowsPerBlock)), block(kRowsPerBlock * 32);
        auto go = [&](auto kern) -> cudaError_t {
            if (rows_smem > 48 * 1024) {
                const cudaError_t e =
                    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(rows_smem));
                if (e != cudaSuccess) return e;
            }
            return launch_pdl(kern, grid, block, rows_smem, s, static_cast<const T *>(x), cin,
                              static_cast<const T *>(w), cout, mv, static_cast<T *>(y), d_status);
        };
        LAT_CUDA_TRY(wt ? go(conv_rows_kernel<T, true>) : go(conv_rows_kernel<T, false>));
        return LAT_OK;
    }
    const size_t smem = sizeof(float) * size_t(cin) * kCoChunk;
    if (wt)
        LAT_CUDA_TRY(launch_pdl(conv_simt_kernel<T, true>, dim3(unsigned(mv.ntiles)), dim3(LAT_TILE_ROWS), smem, s,
                                static_cast<const T *>(x), cin, static_cast<const T *>(w), cout, mv,
                                static_cast<T *>(y), d_status));
    else
        LAT_CUDA_TRY(launch_pdl(conv_simt_kernel<T, false>, dim3(unsigned(mv.ntiles)), dim3(LAT_TILE_ROWS), smem, s,
                                static_cast<const T *>(x), cin, static_cast<const T *>(w), cout, mv,
                                static_cast<T *>(y), d_status));
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
    const int64_t units_max = (map->pair_capacity + kWgradChunkSimt - 1) / kWgradChunkSimt + map->k3;
    Carver cv(ws);
    int32_t *unit_base = cv.take<int32_t>(size_t(map->k3) + 1);
    float *partial = cv.take<float>(size_t(units_max) * cin * cout);
    LAT_CUDA_TRY(launch_pdl(wgrad_units_kernel, dim3(1), dim3(32), 0, s, map->pair_off, map->k3, map->pair_capacity,
                            kWgradChunkSimt, unit_base));
    LAT_CUDA_TRY(cudaGetLastError());
    const int64_t nslices = (int64_t(cin) * cout + kWgradSlice - 1) / kWgradSlice;
    const int64_t parts = nslices >= kWgradWarps ? 1 : (kWgradWarps % nslices == 0 ? kWgradWarps / nslices : 1);
    const int64_t per_block = kWgradWarps / parts;
    const int64_t grid = units_max * ((nslices + per_block - 1) / per_block);
    if (grid >= (int64_t(1) << 31)) return LAT_ERR_UNSUPPORTED;
    LAT_CUDA_TRY(launch_pdl(wgrad_simt_kernel<T>, dim3(unsigned(grid)), dim3(kWgradWarps * 32), 0, s,
                            static_cast<const T *>(x), cin, static_cast<const T *>(dy), cout, map->pair_off,
                            map->pair_in, map->pair_out, map->pair_capacity, map->k3, map->n_in, map->n_out, unit_base,
                            kWgradChunkSimt, partial, d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    const int nelem = cin * cout;
    dim3 rg((nelem + 255) / 256, map->k3);
    LAT_CUDA_TRY(launch_pdl(wgrad_reduce_kernel, dim3(rg), dim3(256), 0, s, partial, unit_base, map->k3, nelem, dw));
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
