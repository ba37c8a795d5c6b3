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
// Weight gradient: the pair list is cut into a fixed number of shares; every
// (share, offset) segment is reduced into one fp32 partial, then the partials
// of each offset are summed in share order, so the result is deterministic.
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

// ----------------------------------------------------------------------------- weight gradient
// dW[k] = sum over the pairs (i, j) of offset k of x[i]^T dy[j].  The pair list
// (grouped by offset) is cut into S equal contiguous shares -- S a constant of
// the channel counts, so the cut depends on neither the GPU nor the buffer
// sizes -- and each share into segments, its intersections with the offsets'
// pair ranges.  A segment's sum is written as one fp32 partial at slot
// share + offset (unique: shares and offsets are both in pair order, so along
// the pair list every step moves to a later share or a later offset); a
// second kernel adds the partials of each offset in share order.  Every sum
// runs in a fixed order, so dW is deterministic, and the scratch holds
// (S + k3) partials whatever the pair count.
constexpr int kSharesLanes = 1184;  // small Cin x Cout (register-tiled kernel)
constexpr int kSharesSlices = 296;  // large Cin x Cout (slice kernel)
constexpr int kLanesMaxElems = 2048;  // Cin x Cout handled by the register-tiled kernel (<= 32 8x8 tiles)

// Shares actually used for P pairs: at most S_max, and at most P so that no
// share is empty (each share writes the partials its slots stand for).
__device__ __forceinline__ int share_count(int64_t P, int s_max) { return int(min(int64_t(s_max), P)); }
__device__ __forceinline__ int64_t share_lo(int64_t P, int v, int S) { return P * v / S; }

// The share holding pair `pair` (largest v with share_lo(P, v) <= pair).
__device__ __forceinline__ int share_of(int64_t P, int64_t pair, int S) {
    int lo = 0, hi = S - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (share_lo(P, mid, S) <= pair) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Register-tiled weight gradient for Cin x Cout <= 2048: the partial is cut
// into 8x8 tiles (input channels ci0..ci0+7, output channels co0..co0+7), E of
// them, and LP = E rounded up to a power of two lanes share one pair: lane
// (q, t) takes tile t of every PW = 32 / LP-th pair, loads its 8 x values and
// 8 dy values (16- or 32-byte loads) and does 64 FMAs, so one warp covers PW
// pairs per step and a block 8 PW.  At the end of a segment the PW lanes of
// each tile are summed with a fixed butterfly, the 8 warps' sums are added in
// warp order through shared memory (E x 64 floats per warp), and the result
// is stored as the segment's partial.  Persistent blocks walk the shares
// blockIdx.x, + gridDim.x, ...
template <typename T>
__global__ void __launch_bounds__(256)
wgrad_lanes_kernel(const T *__restrict__ x, int cin, const T *__restrict__ dy, int cout,
                   const int64_t *__restrict__ pair_off, const int32_t *__restrict__ pair_in,
                   const int32_t *__restrict__ pair_out, int64_t capacity, int k3, int64_t n_in, int64_t n_out,
                   float *__restrict__ partial, int32_t *d_status) {
    pdl_enter();
    extern __shared__ float s_red[];  // [8 warps][E * 64]
    __shared__ int64_t s_off[33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cob = cout / 8, E = (cin / 8) * cob;
    int LP = 1;
    while (LP < E) LP <<= 1;
    const int PW = 32 / LP;
    const int tq = lane % LP, q = warp * PW + lane / LP, step = 8 * PW;
    const bool tile_ok = tq < E;
    const int ci0 = tile_ok ? (tq / cob) * 8 : 0, co0 = tile_ok ? (tq % cob) * 8 : 0;
    if (threadIdx.x <= k3) s_off[threadIdx.x] = min(pair_off[threadIdx.x], capacity);
    __syncthreads();
    const int64_t P = s_off[k3];
    const int S = share_count(P, kSharesLanes);
    const int nelem = cin * cout;
    int32_t bad = 0;
    for (int v = blockIdx.x; v < S; v += gridDim.x) {
        int64_t lo = share_lo(P, v, S);
        const int64_t hi = share_lo(P, v + 1, S);
        int k = 0;
        while (k < k3 && s_off[k + 1] <= lo) ++k;
        while (lo < hi) {
            const int64_t seg_hi = min(hi, s_off[k + 1]);
            float acc[8][8];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
            if (tile_ok) {
                for (int64_t p0 = lo + q; p0 < seg_hi; p0 += 2 * step) {
                    float xv[2][8], gv[2][8];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int64_t p = p0 + u * step;
                        int i = -1, jj = -1;
                        if (p < seg_hi) {
                            i = __ldg(pair_in + p);
                            jj = __ldg(pair_out + p);
                            if (i < 0 || i >= n_in || jj < 0 || jj >= n_out) {
                                bad |= LAT_ERR_BAD_MAP;
                                i = jj = -1;
                            }
                        }
                        if (i >= 0) {
                            load8<T>(x + int64_t(i) * cin + ci0, xv[u]);
                            load8<T>(dy + int64_t(jj) * cout + co0, gv[u]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; ++c) xv[u][c] = gv[u][c] = 0.f;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int a = 0; a < 8; ++a)
#pragma unroll
                            for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(xv[u][a], gv[u][b], acc[a][b]);
                }
            }
            // lanes of one tile: a fixed butterfly over the pair lanes
            for (int o = LP; o < 32; o <<= 1)
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[a][b] += __shfl_xor_sync(0xFFFFFFFFu, acc[a][b], o);
            if (lane < LP && tile_ok) {
                float *dst = s_red + (warp * E + tq) * 64;
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; b += 4)
                        *reinterpret_cast<float4 *>(dst + a * 8 + b) =
                            make_float4(acc[a][b], acc[a][b + 1], acc[a][b + 2], acc[a][b + 3]);
            }
            __syncthreads();
            // the 8 warps' sums in warp order, stored row-major (ci, co) at slot v + k
            float *out = partial + int64_t(v + k) * nelem;
            for (int e = threadIdx.x; e < E * 64; e += blockDim.x) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) sum += s_red[w * E * 64 + e];
                const int tt = e / 64, a = (e % 64) / 8, b = e % 8;
                out[((tt / cob) * 8 + a) * cout + (tt % cob) * 8 + b] = sum;
            }
            __syncthreads();
            lo = seg_hi;
            ++k;
            while (k < k3 && s_off[k + 1] <= lo) ++k;
        }
    }
    if (bad) flag(d_status, bad);
}

// Slice weight gradient for Cin x Cout > 2048: a slice is 256 consecutive
// elements of the Cin x Cout partial; lane l owns 8 consecutive output
// channels of one input channel, so for every pair all 32 lanes read the same
// x row (one value each) and the same dy row (one 32-byte piece each) --
// coalesced, broadcast loads -- and do 8 FMAs.  Block (share v, group of 8
// slices): each warp takes one slice over every segment of the share, pairs
// in order, 4 at a time.
constexpr int kWgradSlice = 256;
constexpr int kWgradWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kWgradWarps * 32)
wgrad_slices_kernel(const T *__restrict__ x, int cin, const T *__restrict__ dy, int cout,
                    const int64_t *__restrict__ pair_off, const int32_t *__restrict__ pair_in,
                    const int32_t *__restrict__ pair_out, int64_t capacity, int k3, int64_t n_in, int64_t n_out,
                    float *__restrict__ partial, int32_t *d_status) {
    pdl_enter();
    __shared__ int64_t s_off[33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nelem = cin * cout;
    const int nslices = (nelem + kWgradSlice - 1) / kWgradSlice;
    const int groups = (nslices + kWgradWarps - 1) / kWgradWarps;
    const int v = blockIdx.x / groups;
    const int slice = (blockIdx.x % groups) * kWgradWarps + warp;
    const int e0 = slice * kWgradSlice + lane * 8;
    const bool own = slice < nslices && e0 < nelem;
    const int ci = own ? e0 / cout : 0, co0 = own ? e0 % cout : 0;
    if (threadIdx.x <= k3) s_off[threadIdx.x] = min(pair_off[threadIdx.x], capacity);
    __syncthreads();
    const int64_t P = s_off[k3];
    const int S = share_count(P, kSharesSlices);
    if (v >= S) return;
    int64_t lo = share_lo(P, v, S);
    const int64_t hi = share_lo(P, v + 1, S);
    int k = 0;
    while (k < k3 && s_off[k + 1] <= lo) ++k;
    int32_t bad = 0;
    while (lo < hi) {
        const int64_t seg_hi = min(hi, s_off[k + 1]);
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
        if (own) {
            for (int64_t p0 = lo; p0 < seg_hi; p0 += 4) {
                float xv[4], gv[4][8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t p = p0 + u;
                    int i = -1, jj = -1;
                    if (p < seg_hi) {
                        i = __ldg(pair_in + p);
                        jj = __ldg(pair_out + p);
                        if (i < 0 || i >= n_in || jj < 0 || jj >= n_out) {
                            bad |= LAT_ERR_BAD_MAP;
                            i = jj = -1;
                        }
                    }
                    xv[u] = 0.f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) gv[u][c] = 0.f;
                    if (i >= 0) {
                        xv[u] = Elem<T>::to_f(x[int64_t(i) * cin + ci]);
                        load8<T>(dy + int64_t(jj) * cout + co0, gv[u]);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[c] = fmaf(xv[u], gv[u][c], acc[c]);
            }
            float *dst = partial + int64_t(v + k) * nelem + e0;
            reinterpret_cast<float4 *>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        lo = seg_hi;
        ++k;
        while (k < k3 && s_off[k + 1] <= lo) ++k;
    }
    if (bad) flag(d_status, bad);
}

// dW[k] = the partials of offset k's segments (0 for an offset without
// pairs).  s_max: the share count the main kernel was given.  R consecutive
// lanes (a power of two <= 32) take one element: lane l adds shares v0+l,
// v0+l+R, ... in order, then an xor butterfly over the R lanes adds the lane
// sums in a fixed tree.  R depends only on the shapes (wgrad_reduce_lanes), so
// the order, and the result, is the same on every call.
__global__ void __launch_bounds__(256)
wgrad_share_reduce_kernel(const float *__restrict__ partial, const int64_t *__restrict__ pair_off, int64_t capacity,
                          int k3, int nelem, int s_max, int lanes, float *__restrict__ dw) {
    pdl_enter();
    __shared__ int s_v[2];
    const int k = blockIdx.y;
    if (threadIdx.x == 0) {
        const int64_t P = min(pair_off[k3], capacity);
        const int S = share_count(P, s_max);
        const int64_t lo = min(pair_off[k], capacity), hi = min(pair_off[k + 1], capacity);
        s_v[0] = lo < hi ? share_of(P, lo, S) : 0;
        s_v[1] = lo < hi ? share_of(P, hi - 1, S) : -1;
    }
    __syncthreads();
    const int l = threadIdx.x & (lanes - 1);
    const int el = (blockIdx.x * blockDim.x + threadIdx.x) / lanes;
    float acc = 0.f;
    if (el < nelem) {
#pragma unroll 4
        for (int v = s_v[0] + l; v <= s_v[1]; v += lanes) acc += partial[int64_t(v + k) * nelem + el];
    }
    for (int m = 1; m < lanes; m <<= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, m);
    if (l == 0 && el < nelem) dw[int64_t(k) * nelem + el] = acc;
}

// Lanes per element of the reduce: about four partials per lane for an
// offset that meets the average number of shares.
static int wgrad_reduce_lanes(int s_max, int k3) {
    int r = 1;
    while (r < 32 && 8 * r <= s_max / k3) r <<= 1;
    return r;
}

// ----------------------------------------------------------------------------- host side
static int wgrad_shares(int cin, int cout) {
    return int64_t(cin) * cout <= kLanesMaxElems ? kSharesLanes : kSharesSlices;
}

size_t wgrad_simt_ws_bytes(int cin, int cout, const lat_kmap *map) {
    return align_up(sizeof(float) * size_t(wgrad_shares(cin, cout) + map->k3) * size_t(cin) * size_t(cout), 256);
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
    float *partial = static_cast<float *>(ws);
    const int nelem = cin * cout;
    const int S = wgrad_shares(cin, cout);
    if (nelem <= kLanesMaxElems) {
        const int E = (cin / 8) * (cout / 8);
        const size_t smem = sizeof(float) * 8 * size_t(E) * 64;
        auto kern = wgrad_lanes_kernel<T>;
        if (smem > 48 * 1024)
            LAT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
        const int grid = std::min(S, 2 * num_sms());
        LAT_CUDA_TRY(launch_pdl(kern, dim3(grid), dim3(256), smem, s, static_cast<const T *>(x), cin,
                                static_cast<const T *>(dy), cout, map->pair_off, map->pair_in, map->pair_out,
                                map->pair_capacity, map->k3, map->n_in, map->n_out, partial, d_status));
    } else {
        const int nslices = (nelem + kWgradSlice - 1) / kWgradSlice;
        const int groups = (nslices + kWgradWarps - 1) / kWgradWarps;
        LAT_CUDA_TRY(launch_pdl(wgrad_slices_kernel<T>, dim3(unsigned(S * groups)), dim3(kWgradWarps * 32), 0, s,
                                static_cast<const T *>(x), cin, static_cast<const T *>(dy), cout, map->pair_off,
                                map->pair_in, map->pair_out, map->pair_capacity, map->k3, map->n_in, map->n_out,
                                partial, d_status));
    }
    LAT_CUDA_TRY(cudaGetLastError());
    const int lanes = wgrad_reduce_lanes(S, map->k3);
    const dim3 rg(unsigned((int64_t(nelem) * lanes + 255) / 256), map->k3);
    LAT_CUDA_TRY(launch_pdl(wgrad_share_reduce_kernel, rg, dim3(256), 0, s, partial, map->pair_off, map->pair_capacity,
                            map->k3, nelem, S, lanes, dw));
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
