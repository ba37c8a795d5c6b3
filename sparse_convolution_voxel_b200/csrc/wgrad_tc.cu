// tcgen05 per-offset weight gradient: dW[k] = sum over pairs (i, j) of offset k of
// x[i]^T dy[j]  (fp16 / bf16 in, fp32 accumulate in TMEM, fp32 out).
//
// Per offset this is a GEMM with M = Cin, N = Cout and the pairs as the
// reduction dimension.  The pairs of each offset (grouped and ordered by the
// kernel-map query) are cut into chunks whose size depends only on the total
// pair count P (chunk_pairs: about kTargetUnits chunks in all, whatever the
// GPU); persistent CTAs (two per SM) take chunks round-robin.  For every
// 64-pair block of a chunk, four gather warps copy the 64 x rows and 64 dy
// rows with 16-byte cp.async into 128-byte swizzled MN-major tiles (rows of
// the gathered operands are the reduction dimension, channels are
// contiguous); the copies arrive on the stage barrier by themselves
// (cp.async.mbarrier.arrive.noinc), and one thread issues 4 tcgen05.mma
// (K = 16 pairs each) into a TMEM accumulator.  Four epilogue warps write the
// chunk's fp32 partial; a second kernel sums the partials of each offset in a
// fixed order (32 interleaved lanes over the chunks, then the lanes in order).
// No atomics, so dW is deterministic and does not depend on the SM count.
#include "common.cuh"
#include "conv_common.cuh"
#include "tc_ptx.cuh"

namespace lat {
namespace wtc {

constexpr int kKP = 64;            // pairs per stage (GEMM K block)
constexpr int kTargetUnits = 448;  // chunks of all offsets together, about
constexpr int kMinChunk = 256;     // pairs per chunk at least
constexpr int kProdWarps = 4, kEpiWarps = 4;
constexpr int kMmaWarp = kProdWarps + kEpiWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr uint64_t kWaitNs = 2000000000ull;

template <int M, int N>
struct Cfg {
    static constexpr uint32_t kABytes = uint32_t(M) * 128;  // 64 pairs x M channels x 2 bytes
    static constexpr uint32_t kBBytes = uint32_t(N) * 128;
    static constexpr uint32_t kStage = kABytes + kBBytes;
    // about 96 KB of stages so that two CTAs share an SM
    static constexpr int kStages = kStage <= 16384 ? 6 : (kStage <= 24576 ? 4 : 3);
    static constexpr uint32_t kSmem = kStages * kStage + 256 + 1024;
    static constexpr uint32_t kTmemCols = 2 * N;
};

template <typename T> constexpr bool is_bf16() { return !std::is_same<T, __half>::value; }

template <typename T, int M, int N> struct KernelTag {};  // one launch-config cache per kernel

// kind::f16, fp32 D, A and B MN-major, M x N
template <typename T, int M, int N>
__host__ __device__ constexpr uint32_t make_idesc() {
    return (1u << 4) | ((is_bf16<T>() ? 1u : 0u) << 7) | ((is_bf16<T>() ? 1u : 0u) << 10) | (1u << 15) |
           (1u << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Pairs per chunk for P pairs in all: at least kMinChunk, a multiple of 64, and
// large enough that the chunks of all offsets number at most kTargetUnits + k3.
__host__ __device__ __forceinline__ int64_t chunk_pairs(int64_t P) {
    const int64_t c = (P + kTargetUnits - 1) / kTargetUnits;
    const int64_t r = (c + 63) / 64 * 64;
    return r > kMinChunk ? r : kMinChunk;
}

// First unit of every offset (and the total in ub[k3]): offset k's clamped pairs
// are cut into ceil(P_k / chunk) units, numbered in offset order; ub[k3 + 1] =
// chunk.  Called by one full warp (lane k handles offset k, k3 <= 32).
__device__ __forceinline__ void unit_bases(const int64_t *pair_off, int64_t capacity, int k3, int32_t *ub) {
    const int lane = threadIdx.x & 31;
    const int64_t P = min(pair_off[k3], capacity);
    const int64_t chunk = chunk_pairs(P);
    const int64_t lo = lane < k3 ? min(pair_off[lane], capacity) : P;
    const int64_t up = __shfl_down_sync(0xFFFFFFFFu, lo, 1);
    const int64_t hi = lane == 31 ? P : up;  // offset k ends where offset k+1 starts (P after the last)
    const int32_t units = lane < k3 ? int32_t((hi - lo + chunk - 1) / chunk) : 0;
    int32_t incl = units;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
    }
    if (lane < k3) ub[lane] = incl - units;
    const int32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (lane == 0) {
        ub[k3] = total;
        ub[k3 + 1] = int32_t(chunk);
    }
}

// Unit u covers pairs [lo, hi) of offset k.
__device__ __forceinline__ void unit_range(const int32_t *unit_base, const int64_t *pair_off, int64_t capacity,
                                           int k3, int32_t u, int &k, int64_t &lo, int64_t &hi) {
    const int64_t chunk = unit_base[k3 + 1];
    k = 0;
    while (k + 1 < k3 && unit_base[k + 1] <= u) ++k;
    const int64_t base = min(pair_off[k], capacity);
    lo = base + int64_t(u - unit_base[k]) * chunk;
    hi = min(lo + chunk, min(pair_off[k + 1], capacity));
}

template <typename T, int M, int N>
__global__ void __launch_bounds__(kThreads, 2)
wgrad_tc_kernel(const T *__restrict__ x, const T *__restrict__ dy, const int64_t *__restrict__ pair_off,
                const int32_t *__restrict__ pair_in, const int32_t *__restrict__ pair_out, int64_t capacity, int k3,
                int64_t n_in, int64_t n_out, float *__restrict__ partial, int32_t *d_status) {
    using C = Cfg<M, N>;
    constexpr int NS = C::kStages;
    constexpr uint32_t idesc = make_idesc<T, M, N>();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NS * C::kStage);
    uint64_t *empty = full + NS;
    uint64_t *accfull = empty + NS;
    uint64_t *accempty = accfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accempty + 2);
    __shared__ int s_abort;
    __shared__ int32_t unit_base[34];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 1) unit_bases(pair_off, capacity, k3, unit_base);
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], kProdWarps * 32);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&accfull[a], 1);
            ptx::mbar_init(&accempty[a], kEpiWarps * 32);
        }
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int32_t units = unit_base[k3];
    int32_t bad = 0;

    if (warp < kProdWarps) {
        // ------------------------------------------------------------ gather x and dy rows
        uint32_t it = 0;
        bool ok = true;
        const int g = lane >> 3, c = lane & 7;
        for (int32_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int k;
            int64_t lo, hi;
            unit_range(unit_base, pair_off, capacity, k3, u, k, lo, hi);
            // lanes 0..15 fetch the indices of this warp's 16 pairs of a block, one block ahead
            auto fetch = [&](int64_t p0, int &si, int &sj) {
                const int64_t mp = p0 + warp * 16 + (lane & 15);
                si = sj = -1;
                if (lane < 16 && mp < hi) {
                    si = __ldg(pair_in + mp);
                    sj = __ldg(pair_out + mp);
                }
            };
            int si_n, sj_n;
            fetch(lo, si_n, sj_n);
            for (int64_t p0 = lo; p0 < hi; p0 += kKP) {
                int si = si_n, sj = sj_n;
                if (p0 + kKP < hi) fetch(p0 + kKP, si_n, sj_n);
                if (si >= n_in || sj >= n_out || (si < 0) != (sj < 0)) {
                    bad |= LAT_ERR_BAD_MAP;
                    si = sj = -1;
                }
                const uint32_t s = it % NS;
                if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, kWaitNs))) {
                    ok = false;
                    break;
                }
                uint8_t *As = smem + s * C::kStage;
                uint8_t *Bs = As + C::kABytes;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pl = 4 * i + g;           // pair within this warp's 16
                    const int p = warp * 16 + pl;       // pair within the 64-pair block (K index)
                    const int ii = __shfl_sync(0xFFFFFFFFu, si, pl);
                    const int jj = __shfl_sync(0xFFFFFFFFu, sj, pl);
                    const uint32_t off = (p >> 3) * 1024 + (p & 7) * 128 + ((c ^ (p & 7)) << 4);
#pragma unroll
                    for (int mb = 0; mb < M / 64; ++mb) {
                        const T *src = ii >= 0 ? x + int64_t(ii) * M + mb * 64 + c * 8 : x;
                        ptx::cp_async16(As + mb * 8192 + off, src, ii >= 0 ? 16u : 0u);
                    }
#pragma unroll
                    for (int nb = 0; nb < N / 64; ++nb) {
                        const T *src = jj >= 0 ? dy + int64_t(jj) * N + nb * 64 + c * 8 : dy;
                        ptx::cp_async16(Bs + nb * 8192 + off, src, jj >= 0 ? 16u : 0u);
                    }
                }
                ptx::cp_async_arrive_noinc(&full[s]);
                ++it;
            }
        }
        ptx::cp_async_wait<0>();
        if (!ok) s_abort = 1;
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------------ epilogue: partial of each unit
        const int q = warp & 3;
        // M = 128: lane l of warp q holds row 32q + l; M = 64: lanes 0..15 hold rows 16q + l
        const int row = M == 128 ? q * 32 + lane : q * 16 + lane;
        const bool has_row = M == 128 || lane < 16;
        uint32_t ta = 0;
        bool ok = true;
        for (int32_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int k;
            int64_t lo, hi;
            unit_range(unit_base, pair_off, capacity, k3, u, k, lo, hi);
            float *dst = partial + int64_t(u) * M * N + int64_t(row) * N;
            if (hi <= lo) {  // cannot happen for a listed unit; keep the partial defined anyway
                if (has_row)
                    for (int c0 = 0; c0 < N; c0 += 4) *reinterpret_cast<float4 *>(dst + c0) = make_float4(0, 0, 0, 0);
                continue;
            }
            const uint32_t a = ta & 1;
            if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(&accfull[a], (ta >> 1) & 1, kWaitNs))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + a * N;
#pragma unroll
            for (int c0 = 0; c0 < N; c0 += 32) {
                uint32_t v0[16], v1[16];
                ptx::tmem_ld16(taddr + c0, v0);
                ptx::tmem_ld16(taddr + c0 + 16, v1);
                ptx::tmem_wait_ld();
                if (has_row) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + c0);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        d4[e] = make_float4(__uint_as_float(v0[4 * e]), __uint_as_float(v0[4 * e + 1]),
                                            __uint_as_float(v0[4 * e + 2]), __uint_as_float(v0[4 * e + 3]));
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        d4[4 + e] = make_float4(__uint_as_float(v1[4 * e]), __uint_as_float(v1[4 * e + 1]),
                                                __uint_as_float(v1[4 * e + 2]), __uint_as_float(v1[4 * e + 3]));
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&accempty[a]);
            ++ta;
        }
        if (!ok) s_abort = 1;
    } else if (lane == 0) {
        // ------------------------------------------------------------ MMA issue
        uint32_t it = 0, ta = 0;
        bool ok = true;
        for (int32_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int k;
            int64_t lo, hi;
            unit_range(unit_base, pair_off, capacity, k3, u, k, lo, hi);
            if (hi <= lo) continue;
            const uint32_t a = ta & 1;
            if (!ptx::mbar_wait(&accempty[a], ((ta >> 1) & 1) ^ 1, kWaitNs)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t dcol = tmem_base + a * N;
            uint32_t acc = 0;
            for (int64_t p0 = lo; p0 < hi; p0 += kKP) {
                const uint32_t s = it % NS;
                if (!ptx::mbar_wait(&full[s], (it / NS) & 1, kWaitNs)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                // the gathered rows were written by cp.async (generic proxy);
                // order them before the tensor core's async-proxy reads
                ptx::fence_proxy_async_smem();
                const uint32_t as = ptx::smem_u32(smem + s * C::kStage);
                const uint32_t bs = as + C::kABytes;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = ptx::desc_sw128(as + ks * 2048, 8192, 1024);
                    const uint64_t bd = ptx::desc_sw128(bs + ks * 2048, 8192, 1024);
                    ptx::umma_f16(dcol, ad, bd, idesc, acc);
                    acc = 1;
                }
                ptx::umma_commit(&empty[s]);
                ++it;
            }
            if (!ok) break;
            ptx::umma_commit(&accfull[a]);
            ++ta;
        }
        if (!ok) s_abort = 1;
    }

    __syncthreads();
    if (s_abort) {
        bad |= (tid == 0) ? LAT_ERR_TIMEOUT : 0;
        __nanosleep(1000000);
    }
    if (bad) flag(d_status, bad);
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// dW[k] = sum of offset k's chunk partials.  Block (x, k): 32 unit lanes x 8
// groups of 4 elements; lane l sums chunks l, l+32, ... in order, then lane 0
// adds the 32 lane sums in order -- a fixed order whatever the timing.
constexpr int kRedLanes = 32;
__global__ void __launch_bounds__(256)
wgrad_tc_reduce_kernel(const float *__restrict__ partial, const int64_t *__restrict__ pair_off, int64_t capacity,
                       int k3, int nelem, float *__restrict__ dw) {
    __shared__ int32_t unit_base[34];
    __shared__ float4 s_part[kRedLanes][8];
    if (threadIdx.x < 32) unit_bases(pair_off, capacity, k3, unit_base);
    __syncthreads();
    const int k = blockIdx.y;
    const int g = threadIdx.x & 7, l = threadIdx.x >> 3;
    const int el = (blockIdx.x * 8 + g) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (el < nelem) {
#pragma unroll 4
        for (int32_t u = unit_base[k] + l; u < unit_base[k + 1]; u += kRedLanes) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(partial + int64_t(u) * nelem + el));
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
    }
    s_part[l][g] = acc;
    __syncthreads();
    if (l == 0 && el < nelem) {
        float4 t = s_part[0][g];
        for (int q = 1; q < kRedLanes; ++q) {
            const float4 v = s_part[q][g];
            t.x += v.x;
            t.y += v.y;
            t.z += v.z;
            t.w += v.w;
        }
        *reinterpret_cast<float4 *>(dw + int64_t(k) * nelem + el) = t;
    }
}

template <typename T, int M, int N>
static lat_status launch(const void *x, const void *dy, const lat_kmap *map, float *dw, void *ws, int32_t *d_status,
                         cudaStream_t s) {
    using C = Cfg<M, N>;
    const int64_t units_max = int64_t(kTargetUnits) + map->k3;
    Carver cv(ws);
    float *partial = cv.take<float>(size_t(units_max) * M * N);
    auto kern = wgrad_tc_kernel<T, M, N>;
    const int64_t grid = std::min<int64_t>(units_max, GridCache<KernelTag<T, M, N>>::get(kern, C::kSmem, int(C::kTmemCols), 2));
    if (grid <= 0) return LAT_ERR_CUDA;
    kern<<<unsigned(grid), kThreads, C::kSmem, s>>>(static_cast<const T *>(x), static_cast<const T *>(dy),
                                                    map->pair_off, map->pair_in, map->pair_out, map->pair_capacity,
                                                    map->k3, map->n_in, map->n_out, partial, d_status);
    LAT_CUDA_TRY(cudaGetLastError());
    const int nelem = M * N;
    dim3 rg((nelem + 31) / 32, map->k3);
    wgrad_tc_reduce_kernel<<<rg, 256, 0, s>>>(partial, map->pair_off, map->pair_capacity, map->k3, nelem, dw);
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

}  // namespace wtc

bool wgrad_tc_supported(int cin, int cout) { return (cin == 64 || cin == 128) && (cout == 64 || cout == 128); }

size_t wgrad_tc_ws_bytes(int cin, int cout, const lat_kmap *map) {
    const int64_t units_max = int64_t(wtc::kTargetUnits) + map->k3;
    Carver cv(nullptr);
    cv.take<float>(size_t(units_max) * cin * cout);
    return align_up(cv.used, 256);
}

lat_status launch_wgrad_tc(bool bf16, const void *x, int cin, const void *dy, int cout, const lat_kmap *map, float *dw,
                           void *ws, int32_t *d_status, cudaStream_t s) {
#define LAT_WTC(T, M, N) \
    if (cin == M && cout == N) return wtc::launch<T, M, N>(x, dy, map, dw, ws, d_status, s);
    if (bf16) {
        LAT_WTC(__nv_bfloat16, 64, 64) LAT_WTC(__nv_bfloat16, 64, 128) LAT_WTC(__nv_bfloat16, 128, 64)
        LAT_WTC(__nv_bfloat16, 128, 128)
    } else {
        LAT_WTC(__half, 64, 64) LAT_WTC(__half, 64, 128) LAT_WTC(__half, 128, 64) LAT_WTC(__half, 128, 128)
    }
#undef LAT_WTC
    return LAT_ERR_UNSUPPORTED;
}

}  // namespace lat
