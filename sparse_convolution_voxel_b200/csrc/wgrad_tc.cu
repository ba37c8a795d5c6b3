// tcgen05 per-offset weight gradient: dW[k] = sum over pairs (i, j) of offset k of
// x[i]^T dy[j]  (fp16 / bf16 in, fp32 accumulate in TMEM, fp32 out).
//
// Per offset this is a GEMM with M = Cin, N = Cout and the pairs as the
// reduction dimension.  The pair list (grouped by offset by the kernel-map
// query) is cut into kWorkers equal contiguous shares (fewer when there are
// fewer pairs than that, so that no share is empty) -- a constant, so the
// cut does not depend on the GPU -- and persistent CTAs (two per SM) take the
// shares round-robin.  A share is processed as segments, its intersections
// with the offsets' pair ranges; a segment accumulates in TMEM and ends in one
// fp32 partial, stored at slot share + offset (unique: shares and offsets are
// both in pair order).  For every 64-pair block of a segment, four gather
// warps copy the 64 x rows and 64 dy
// rows with 16-byte cp.async into 128-byte swizzled MN-major tiles (rows of
// the gathered operands are the reduction dimension, channels are
// contiguous); the copies arrive on the stage barrier by themselves
// (cp.async.mbarrier.arrive.noinc), and one thread issues 4 tcgen05.mma
// (K = 16 pairs each) into a TMEM accumulator.  Four epilogue warps write the
// segment's fp32 partial; a second kernel sums the partials of each offset in a
// fixed order (8 interleaved lanes over the shares, then a fixed xor tree).
// No atomics, so dW is deterministic and does not depend on the SM count.
#include "common.cuh"
#include "conv_common.cuh"
#include "tc_ptx.cuh"

namespace lat {
namespace wtc {

constexpr int kKP = 64;            // pairs per stage (GEMM K block)
constexpr int kWorkers = 296;      // equal shares of the pair list (two per B200 SM)
constexpr int kProdWarps = 4, kEpiWarps = 4;
constexpr int kMmaWarp = kProdWarps + kEpiWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr uint64_t kDrainNs = 1000000000ull;  // limit of the waits that drain a CTA that gave up

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

// Clamped pair offsets of the k3 offsets (off[k3] = P) into shared memory; one warp.
__device__ __forceinline__ void load_offsets(const int64_t *pair_off, int64_t capacity, int k3, int64_t *off) {
    for (int e = threadIdx.x & 31; e <= k3; e += 32) off[e] = min(pair_off[e], capacity);
}

// Shares of a list of P pairs: min(kWorkers, P), so that no share is empty
// (every share then writes the partials its slots stand for).
__device__ __forceinline__ int share_count(int64_t P) { return int(min(int64_t(kWorkers), P)); }

// Share v of the pair list: pairs [P v / S, P (v+1) / S), S = share_count(P).
__device__ __forceinline__ int64_t share_lo(int64_t P, int v) { return P * v / share_count(P); }

// The share holding pair `pair` (largest v with share_lo(P, v) <= pair); a binary search.
__device__ __forceinline__ int share_of(int64_t P, int64_t pair) {
    int lo = 0, hi = share_count(P) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (share_lo(P, mid) <= pair) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// The segments of this CTA's shares, in order: share v = blockIdx.x, +gridDim.x,
// ..., and within a share the offsets its range meets.  Every role walks the
// same sequence.
struct Segments {
    const int64_t *off;
    int k3;
    int64_t P;
    int v, k;
    int64_t hv;
    __device__ Segments(const int64_t *o, int k3_) : off(o), k3(k3_), P(o[k3_]), v(int(blockIdx.x) - int(gridDim.x)),
                                                   k(k3_), hv(0) {}
    // next segment: offset ko, pairs [lo, hi), partial slot
    __device__ bool next(int &ko, int64_t &lo, int64_t &hi, int &slot) {
        for (;;) {
            while (k < k3 && off[k] < hv) {
                const int64_t a = max(share_lo(P, v), off[k]), b = min(hv, off[k + 1]);
                const int kk = k++;
                if (a < b) {
                    ko = kk;
                    lo = a;
                    hi = b;
                    slot = v + kk;
                    return true;
                }
            }
            v += gridDim.x;
            if (v >= share_count(P)) return false;
            const int64_t wl = share_lo(P, v);
            hv = share_lo(P, v + 1);
            k = 0;
            while (k < k3 && off[k + 1] <= wl) ++k;
        }
    }
};

template <typename T, int M, int N>
__global__ void __launch_bounds__(kThreads, 2)
wgrad_tc_kernel(const T *__restrict__ x, const T *__restrict__ dy, const int64_t *__restrict__ pair_off,
                const int32_t *__restrict__ pair_in, const int32_t *__restrict__ pair_out, int64_t capacity, int k3,
                int64_t n_in, int64_t n_out, float *__restrict__ partial, int32_t *__restrict__ ranges,
                uint64_t wait_ns, int32_t *d_status) {
    pdl_enter();
    const uint64_t kWaitNs = wait_ns;
    using C = Cfg<M, N>;
    constexpr int NS = C::kStages;
    constexpr uint32_t idesc = make_idesc<T, M, N>();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NS * C::kStage);
    uint64_t *empty = full + NS;
    uint64_t *accfull = empty + NS;
    uint64_t *accempty = accfull + 2;
    uint64_t *drain = accempty + 2;  // tracks the MMAs still in flight when a CTA gives up
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    __shared__ int s_abort;
    __shared__ int64_t s_off[33];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 1) {
        load_offsets(pair_off, capacity, k3, s_off);
        __syncwarp();
        if (blockIdx.x == 0 && lane < k3) {
            // for the reduce: the shares meeting offset lane's pairs [a, b)
            const int64_t P = s_off[k3], a = s_off[lane], b = s_off[lane + 1];
            ranges[2 * lane] = a < b ? share_of(P, a) : 0;
            ranges[2 * lane + 1] = a < b ? share_of(P, b - 1) : -1;
        }
    }
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], kProdWarps * 32);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&accfull[a], 1);
            ptx::mbar_init(&accempty[a], kEpiWarps * 32);
        }
        ptx::mbar_init(drain, 1);
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
    int32_t bad = 0;

    if (warp < kProdWarps) {
        // ------------------------------------------------------------ gather x and dy rows
        uint32_t it = 0;
        bool ok = true;
        const int g = lane >> 3, c = lane & 7;
        Segments seg(s_off, k3);
        int k, slot;
        int64_t lo, hi;
        while (ok && seg.next(k, lo, hi, slot)) {
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
        Segments seg(s_off, k3);
        int k, slot;
        int64_t lo, hi;
        while (ok && seg.next(k, lo, hi, slot)) {
            float *dst = partial + int64_t(slot) * M * N + int64_t(row) * N;
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
        Segments seg(s_off, k3);
        int k, slot;
        int64_t lo, hi;
        while (ok && seg.next(k, lo, hi, slot)) {
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
        // A role gave up: every thread's cp.async copies are complete
        // (cp.async.wait_all above); the MMA thread commits every MMA it issued
        // to `drain` and waits for it (with its own limit) before the TMEM and
        // shared memory are released.
        bad |= (tid == 0) ? LAT_ERR_TIMEOUT : 0;
        if (warp == kMmaWarp && lane == 0) {
            ptx::umma_commit(drain);
            ptx::mbar_wait(drain, 0, kDrainNs);
        }
        __syncthreads();
    }
    if (bad) flag(d_status, bad);
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// dW[k] = sum of offset k's partials, one per share v0..v1 that meets offset k
// (slot share + k; ranges from the main kernel).  Eight consecutive lanes
// share a float4 column of dW[k]: lane l sums shares v0+l, v0+l+8, ... in
// order, then an xor butterfly over the eight lanes adds the lane sums in a
// fixed tree -- the same order whatever the timing.  Offsets without pairs
// get 0.
constexpr int kRedLanes = 8;
constexpr int kRedThreads = 256;
constexpr int kRedCols = kRedThreads / kRedLanes;  // float4 columns of dW[k] per block
__global__ void __launch_bounds__(kRedThreads)
wgrad_tc_reduce_kernel(const float *__restrict__ partial, const int32_t *__restrict__ ranges, int nelem,
                       float *__restrict__ dw) {
    pdl_enter();
    const int k = blockIdx.y;
    const int v0 = __ldg(ranges + 2 * k), v1 = __ldg(ranges + 2 * k + 1);
    const int l = threadIdx.x & (kRedLanes - 1);
    const int el = (blockIdx.x * kRedCols + threadIdx.x / kRedLanes) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (el < nelem) {
#pragma unroll 4
        for (int v = v0 + l; v <= v1; v += kRedLanes) {
            const float4 x = __ldg(reinterpret_cast<const float4 *>(partial + int64_t(v + k) * nelem + el));
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
    }
#pragma unroll
    for (int m = 1; m < kRedLanes; m <<= 1) {
        acc.x += __shfl_xor_sync(0xFFFFFFFFu, acc.x, m);
        acc.y += __shfl_xor_sync(0xFFFFFFFFu, acc.y, m);
        acc.z += __shfl_xor_sync(0xFFFFFFFFu, acc.z, m);
        acc.w += __shfl_xor_sync(0xFFFFFFFFu, acc.w, m);
    }
    if (l == 0 && el < nelem) *reinterpret_cast<float4 *>(dw + int64_t(k) * nelem + el) = acc;
}

template <typename T, int M, int N>
static lat_status launch(const void *x, const void *dy, const lat_kmap *map, float *dw, void *ws, int32_t *d_status,
                         cudaStream_t s) {
    using C = Cfg<M, N>;
    const int64_t units_max = int64_t(kWorkers) + map->k3;
    Carver cv(ws);
    float *partial = cv.take<float>(size_t(units_max) * M * N);
    int32_t *ranges = cv.take<int32_t>(64);
    auto kern = wgrad_tc_kernel<T, M, N>;
    const int64_t grid = std::min<int64_t>(kWorkers, GridCache<KernelTag<T, M, N>>::get(kern, C::kSmem, int(C::kTmemCols), 2));
    if (grid <= 0) return LAT_ERR_CUDA;
    LAT_CUDA_TRY(launch_pdl(kern, dim3(unsigned(grid)), dim3(kThreads), C::kSmem, s, static_cast<const T *>(x),
                            static_cast<const T *>(dy), map->pair_off, map->pair_in, map->pair_out, map->pair_capacity,
                            map->k3, map->n_in, map->n_out, partial, ranges, wait_limit_ns(), d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    const int nelem = M * N;
    dim3 rg((nelem / 4 + kRedCols - 1) / kRedCols, map->k3);
    LAT_CUDA_TRY(launch_pdl(wgrad_tc_reduce_kernel, dim3(rg), dim3(kRedThreads), 0, s, partial, ranges, nelem, dw));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

}  // namespace wtc

bool wgrad_tc_supported(int cin, int cout) { return (cin == 64 || cin == 128) && (cout == 64 || cout == 128); }

size_t wgrad_tc_ws_bytes(int cin, int cout, const lat_kmap *map) {
    const int64_t units_max = int64_t(wtc::kWorkers) + map->k3;
    Carver cv(nullptr);
    cv.take<float>(size_t(units_max) * cin * cout);
    cv.take<int32_t>(64);
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
