// tcgen05 implicit-GEMM sparse convolution: fp16 / bf16 in, fp32 accumulate in TMEM.
//
// Output-stationary implicit GEMM (TorchSparse++ abstract: implicit GEMM
// overlaps computation and memory access; the migration page's "Backend and
// configuration differences" requires every dataflow to give the same result
// for a fixed relation and weight tensor).  Persistent CTAs (two per SM) take
// 128-row tiles of the mask-sorted output order from a device-wide counter,
// heaviest tiles first; for every offset in a tile's mask union and every
// 64-channel K block a CTA
//   - gathers the 128 neighbour rows with 16-byte cp.async into a 128-byte
//     swizzled K-major tile (absent neighbours are zero-filled, no read);
//     each gather thread's copies arrive on the stage barrier by themselves
//     (cp.async.mbarrier.arrive.noinc), so the thread never waits for them,
//   - loads the W[k] slab with TMA (128-byte swizzle, no multicast),
//   - issues 4 tcgen05.mma (M=128, N=Cout, K=16) into a TMEM accumulator.
// Epilogue warps read the accumulator with tcgen05.ld, round once to the
// output type and write each output row exactly once -- no atomics.  The
// accumulator is double buffered in TMEM so the epilogue of tile t overlaps
// the main loop of tile t+1.
//
// Roles (320 threads): warps 0-3 gather (thread 0 also issues TMA), warps 4-7
// epilogue (warp w reads TMEM lanes 32*(w%4)..+31), warp 8 lane 0 issues MMAs,
// warp 9 claims tiles and publishes (tile, mask union, output rows) in a ring
// of shared-memory entries that the other roles read in order.  The rows are
// sorted by neighbour count (ascending), so walking the tiles backwards hands
// out the long tiles first and the one-offset tiles fill the gaps.
// Every mbarrier wait is bounded (lat_set_wait_limit_ns, 2 s by default); a
// wait that gives up flags LAT_ERR_TIMEOUT, and the CTA waits for its
// in-flight TMA loads and MMAs, releases its TMEM and exits.
//
// The same kernel computes the data gradient: the gathered operand is dy, the
// B operand is W[k]^T (K-major view of the same weight slab), and a
// submanifold map is walked with flipped offsets.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "conv_common.cuh"
#include "tc_ptx.cuh"

namespace lat {
namespace tc {

constexpr int kM = 128;          // tile rows = MMA M
constexpr int kProdWarps = 4;    // gather warps
constexpr int kEpiWarps = 4;     // epilogue warps
constexpr int kMmaWarp = kProdWarps + kEpiWarps;
constexpr int kSchedWarp = kMmaWarp + 1;
constexpr int kThreads = (kSchedWarp + 1) * 32;
constexpr int kRing = 8;         // tile entries in flight between the scheduler and the other roles
constexpr int kItems = 14;       // (tile, offset) items in flight between the scheduler and the gather warps
constexpr uint32_t kStgBytes = kEpiWarps * 32 * 32;  // per epilogue warp: 32 rows x 16 output channels
constexpr uint32_t kABytes = kM * 128;  // 128 rows x 64 channels x 2 bytes
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint64_t kDrainNs = 1000000000ull;  // limit of the waits that drain a CTA that gave up

// One claimed tile as the scheduler publishes it.
struct TileEntry {
    int32_t tile;      // tile index, -1 = no more tiles for this CTA
    uint32_t mask;     // union of the tile rows' offset masks (flipped for a flipped map)
    int32_t pad[2];
    int32_t rows[kM];  // output row of every tile row, -1 past n_out
};

// One (tile, offset) item: the offset and the source row of every tile row,
// as the scheduler warp publishes it for the gather warps.
struct ItemEntry {
    int32_t k;         // offset, -1 = no more items for this CTA
    int32_t pad[3];
    int32_t src[kM];   // input row gathered into each tile row, -1 = none (zero row)
};

template <int N>
struct Cfg {
    static constexpr uint32_t kBBytes = uint32_t(N) * 128;  // 64 K x N (or N x 64) x 2 bytes
    static constexpr uint32_t kStage = kABytes + kBBytes;
    static constexpr int kStages = N == 64 ? 4 : 3;  // ~100 KB: two CTAs per SM
    static constexpr uint32_t kRingOff = kStages * kStage;
    static constexpr uint32_t kItemOff = kRingOff + kRing * sizeof(TileEntry);
    static constexpr uint32_t kStgOff = kItemOff + kItems * sizeof(ItemEntry);
    static constexpr uint32_t kBarOff = kStgOff + kStgBytes;
    static constexpr uint32_t kBarBytes = 512;
    static constexpr uint32_t kSmem = kBarOff + kBarBytes + 1024;
    static constexpr uint32_t kTmemCols = 2 * N;
    // the scheduler can run ahead of the slowest reader (the epilogue) by at
    // most stages + 2 tiles; the ring must be deeper than that
    static_assert(kRing >= kStages + 3, "tile ring too shallow");
    static_assert((2 * kStages + 4 + 2 * kRing + 2 * kItems + 1) * 8 + 4 <= kBarBytes, "barrier area");
    // two CTAs per SM: 228 KB of shared memory per SM, 1 KB reserved per CTA, 16 B static
    static_assert(2 * (kSmem + 16 + 1024) <= 228 * 1024, "two CTAs per SM");
};

template <typename T> constexpr bool is_bf16() { return sizeof(T) == 2 && !std::is_same<T, __half>::value; }

template <typename T, int KC, int N, bool BMN> struct KernelTag {};  // one launch-config cache per kernel

// Instruction descriptor, kind::f16: fp32 D, A/B fp16 or bf16, A K-major,
// B MN-major (forward: W[k] is (Cin x Cout), Cout contiguous) or K-major
// (data gradient: W[k]^T viewed as (N=Cin) x (K=Cout) rows), M=128, N.
template <typename T, int N, bool BMN>
__host__ __device__ constexpr uint32_t make_idesc() {
    return (1u << 4) | ((is_bf16<T>() ? 1u : 0u) << 7) | ((is_bf16<T>() ? 1u : 0u) << 10) |
           ((BMN ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(kM >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack2(float a, float b, __half) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// KC: gathered channels (GEMM K), N: output channels, BMN: B operand MN-major.
// tile_counter: zero at launch; CTAs claim tiles past the first gridDim.x from it.
// wait_ns: how long any one barrier wait may take before the CTA gives up.
template <typename T, int KC, int N, bool BMN>
__global__ void __launch_bounds__(kThreads, 2)
conv_tc_kernel(const __grid_constant__ CUtensorMap wmap, const T *__restrict__ x, MapView mv, T *__restrict__ y,
               int32_t *tile_counter, uint64_t wait_ns, int32_t *d_status) {
    const uint64_t kWaitNs = wait_ns;
    pdl_enter();
    using C = Cfg<N>;
    constexpr int NS = C::kStages;
    constexpr int KBLK = KC / 64;
    constexpr uint32_t idesc = make_idesc<T, N, BMN>();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    TileEntry *ring = reinterpret_cast<TileEntry *>(smem + C::kRingOff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + NS;
    uint64_t *accfull = empty + NS;
    uint64_t *accempty = accfull + 2;
    uint64_t *ring_full = accempty + 2;
    uint64_t *ring_empty = ring_full + kRing;
    uint64_t *item_full = ring_empty + kRing;
    uint64_t *item_empty = item_full + kItems;
    uint64_t *drain = item_empty + kItems;  // tracks the MMAs still in flight when a CTA gives up
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    ItemEntry *items = reinterpret_cast<ItemEntry *>(smem + C::kItemOff);
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            // 128 gather threads' copy completions + the weight thread's expect_tx
            ptx::mbar_init(&full[s], kProdWarps * 32 + 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&accfull[a], 1);
            ptx::mbar_init(&accempty[a], kEpiWarps * 32);
        }
        for (int r = 0; r < kRing; ++r) {
            ptx::mbar_init(&ring_full[r], 32);
            ptx::mbar_init(&ring_empty[r], 1 + kEpiWarps * 32);  // MMA thread + epilogue threads
        }
        for (int r = 0; r < kItems; ++r) {
            ptx::mbar_init(&item_full[r], 64);  // 32 index-copy completions + 32 plain arrivals
            ptx::mbar_init(&item_empty[r], kProdWarps * 32);
        }
        ptx::mbar_init(drain, 1);
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
        ptx::tma_prefetch(&wmap);
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool y32 = (reinterpret_cast<uintptr_t>(y) & 31) == 0;  // 256-bit stores of output slices
    int32_t bad = 0;
    uint32_t stages_issued = 0;  // thread 0: stage fills (each with a weight TMA) issued

    if (warp < kProdWarps) {
        // ------------------------------------------------------------ gather + TMA
        // Thread tid owns tile row tid; its source row of every item comes
        // from the item ring, so no global index load sits on this path.
        uint32_t it = 0;
        bool ok = true;
        for (int ii = 0; ok; ++ii) {
            const int r = ii % kItems;
            if (!__all_sync(kFull, ptx::mbar_wait(&item_full[r], (ii / kItems) & 1, kWaitNs))) {
                ok = false;
                break;
            }
            const int k = items[r].k;
            int src_own = items[r].src[tid];
            ptx::mbar_arrive(&item_empty[r]);
            if (k < 0) break;
            if (src_own >= mv.n_in) {
                bad |= LAT_ERR_BAD_MAP;
                src_own = -1;
            }
            for (int kb = 0; kb < KBLK; ++kb) {
                const uint32_t s = it % NS;
                if (!__all_sync(kFull, ptx::mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, kWaitNs))) {
                    ok = false;
                    break;
                }
                uint8_t *As = smem + s * C::kStage;
                uint8_t *Bs = As + kABytes;
                if (tid == 0) {
                    ptx::mbar_arrive_expect_tx(&full[s], C::kBBytes);
#pragma unroll
                    for (int nb = 0; nb < N / 64; ++nb) {
                        if constexpr (BMN)  // rows k*KC + 64kb.., columns 64nb..
                            ptx::tma_load_2d(Bs + nb * 8192, &wmap, &full[s], 64 * nb, k * KC + 64 * kb);
                        else                // rows k*N + 64nb.., columns 64kb..
                            ptx::tma_load_2d(Bs + nb * 8192, &wmap, &full[s], 64 * kb, k * N + 64 * nb);
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rl = 4 * i + (lane >> 3);
                    const int row = warp * 32 + rl;
                    const int chunk = lane & 7;
                    const int src = __shfl_sync(kFull, src_own, rl);
                    const T *gp = src >= 0 ? x + int64_t(src) * KC + kb * 64 + chunk * 8 : x;
                    ptx::cp_async16(As + row * 128 + ((chunk ^ (row & 7)) << 4), gp, src >= 0 ? 16u : 0u);
                }
                ptx::cp_async_arrive_noinc(&full[s]);
                ++it;
            }
        }
        ptx::cp_async_wait<0>();
        stages_issued = it;
        if (!ok) s_abort = 1;
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        uint32_t ta = 0;
        bool ok = true;
        for (int ri = 0; ok; ++ri) {
            const int r = ri % kRing;
            if (!__all_sync(kFull, ptx::mbar_wait(&ring_full[r], (ri / kRing) & 1, kWaitNs))) {
                ok = false;
                break;
            }
            const int t = ring[r].tile;
            const uint32_t tm = ring[r].mask;
            const int j = t >= 0 ? ring[r].rows[q * 32 + lane] : -1;
            ptx::mbar_arrive(&ring_empty[r]);
            if (t < 0) break;
            T *yr = j >= 0 ? y + int64_t(j) * N : nullptr;
            if (!tm) {  // no neighbour anywhere in the tile: zeros
                if (yr)
#pragma unroll
                    for (int c = 0; c < N; c += 8) *reinterpret_cast<uint4 *>(yr + c) = make_uint4(0, 0, 0, 0);
                continue;
            }
            const uint32_t a = ta & 1;
            if (!__all_sync(kFull, ptx::mbar_wait(&accfull[a], (ta >> 1) & 1, kWaitNs))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + a * N;
            // Write-back of each 16-channel slice (32 B of a row).  With a 32-byte
            // aligned output every lane stores its own row's slice with one 256-bit
            // store: a whole 32-byte sector per lane, no staging.  Otherwise the
            // warp's 32 rows go through a 1 KB staging buffer (the two 16-byte
            // halves swapped on every other group of 4 rows against bank
            // conflicts) and lane pairs write whole 32-byte sectors of one row.
            uint8_t *stg = smem + C::kStgOff + q * 1024;
            auto write_slice = [&](const uint32_t (&v)[16], int col) {
                if (y32) {
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o[e] = pack2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]), T{});
                    if (j >= 0) ptx::st_global_v8(y + int64_t(j) * N + col, o);
                    return;
                }
                uint4 o0, o1;
                o0.x = pack2(__uint_as_float(v[0]), __uint_as_float(v[1]), T{});
                o0.y = pack2(__uint_as_float(v[2]), __uint_as_float(v[3]), T{});
                o0.z = pack2(__uint_as_float(v[4]), __uint_as_float(v[5]), T{});
                o0.w = pack2(__uint_as_float(v[6]), __uint_as_float(v[7]), T{});
                o1.x = pack2(__uint_as_float(v[8]), __uint_as_float(v[9]), T{});
                o1.y = pack2(__uint_as_float(v[10]), __uint_as_float(v[11]), T{});
                o1.z = pack2(__uint_as_float(v[12]), __uint_as_float(v[13]), T{});
                o1.w = pack2(__uint_as_float(v[14]), __uint_as_float(v[15]), T{});
                const int sw = (lane >> 2) & 1;
                *reinterpret_cast<uint4 *>(stg + lane * 32 + 16 * sw) = o0;
                *reinterpret_cast<uint4 *>(stg + lane * 32 + 16 * (sw ^ 1)) = o1;
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const int rr = 16 * g + (lane >> 1), hc = lane & 1;
                    const uint4 val =
                        *reinterpret_cast<const uint4 *>(stg + rr * 32 + 16 * (hc ^ ((rr >> 2) & 1)));
                    const int jr = __shfl_sync(kFull, j, rr);
                    if (jr >= 0) *reinterpret_cast<uint4 *>(y + int64_t(jr) * N + col + 8 * hc) = val;
                }
                __syncwarp();
            };
#pragma unroll
            for (int c0 = 0; c0 < N; c0 += 32) {
                uint32_t v0[16], v1[16];
                ptx::tmem_ld16(taddr + c0, v0);
                ptx::tmem_ld16(taddr + c0 + 16, v1);
                ptx::tmem_wait_ld();
                write_slice(v0, c0);
                write_slice(v1, c0 + 16);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&accempty[a]);
            ++ta;
        }
        if (!ok) s_abort = 1;
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            uint32_t it = 0, ta = 0;
            bool ok = true;
            for (int ri = 0; ok; ++ri) {
                const int r = ri % kRing;
                if (!ptx::mbar_wait(&ring_full[r], (ri / kRing) & 1, kWaitNs)) {
                    ok = false;
                    break;
                }
                const int t = ring[r].tile;
                const uint32_t tm = ring[r].mask;
                ptx::mbar_arrive(&ring_empty[r]);
                if (t < 0) break;
                if (!tm) continue;
                const uint32_t a = ta & 1;
                if (!ptx::mbar_wait(&accempty[a], ((ta >> 1) & 1) ^ 1, kWaitNs)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t dcol = tmem_base + a * N;
                uint32_t acc = 0;
                for (uint32_t m = tm; m && ok; m &= m - 1) {
                    for (int kb = 0; kb < KBLK; ++kb) {
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
                        const uint32_t bs = as + kABytes;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t ad = ptx::desc_sw128(as + ks * 32, 16, 1024);
                            const uint64_t bd = BMN ? ptx::desc_sw128(bs + ks * 2048, 8192, 1024)
                                                    : ptx::desc_sw128(bs + ks * 32, 16, 1024);
                            ptx::umma_f16(dcol, ad, bd, idesc, acc);
                            acc = 1;
                        }
                        ptx::umma_commit(&empty[s]);
                        ++it;
                    }
                }
                if (!ok) break;
                ptx::umma_commit(&accfull[a]);
                ++ta;
            }
            if (!ok) s_abort = 1;
        }
    } else {
        // ------------------------------------------------------------ tile scheduler + neighbour indices
        // Claim order q = 0, 1, ...: q < gridDim.x is CTA q's first tile, later q
        // come from the counter; tile = ntiles-1-q (heaviest first).  The mask and
        // output rows of a tile are loaded two tiles ahead; the neighbour indices
        // are copied into the item ring with cp.async, whose completion the item
        // barrier tracks, so this warp never waits for index data.
        bool ok = true;
        int ii = 0;  // items published
        auto fetch = [&](int64_t q, int64_t &t, uint32_t &tm, int (&rows)[4]) {
            t = q < mv.ntiles ? mv.ntiles - 1 - q : -1;
            tm = t >= 0 ? mv.tile_mask_at(t) : 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t row = t * kM + e * 32 + lane;
                rows[e] = (t >= 0 && row < mv.n_out) ? __ldg(mv.perm + row) : -1;
            }
        };
        auto push_item = [&](int k, const int (&rows)[4]) -> bool {
            const int r = ii % kItems;
            if (!__all_sync(kFull, ptx::mbar_wait(&item_empty[r], ((ii / kItems) & 1) ^ 1, kWaitNs))) return false;
            if (lane == 0) items[r].k = k;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int32_t *dst = &items[r].src[e * 32 + lane];
                if (k >= 0 && k == mv.centre)
                    *dst = rows[e];  // submanifold centre: every row is its own neighbour
                else if (k >= 0 && rows[e] >= 0)
                    ptx::cp_async4(dst, mv.neighbour_ptr(k, rows[e]));
                else
                    *dst = -1;
            }
            ptx::cp_async_arrive_noinc(&item_full[r]);
            ptx::mbar_arrive(&item_full[r]);
            ++ii;
            return true;
        };
        // kLook slots of (tile, mask, rows) rotate through the loop: slot s is
        // published, its items pushed, and refilled with a later tile, so each
        // row load has up to kLook-1 tiles of time to land.  The loop over
        // slots is unrolled; no register holding a load in flight is moved.
        // Tile 0 is static; the other slots are first filled once tile 0's
        // items are pushed, so a CTA holding a long tile does not take light
        // tiles early.  Positions come from the counter in batches while the
        // tiles being published are light (at most 2 offsets): 4 while more than
        // 8 tiles per CTA remain, 2 above 2, else 1 (one tile at a time near the
        // end keeps the CTAs balanced); the next batch is claimed when the
        // current one is handed out.
        constexpr int kLook = 3;
        constexpr int64_t kUnfetched = -2;
        int64_t ts[kLook];
        uint32_t ms[kLook];
        int rs[kLook][4];
        bool more = true;      // the counter may still hold tiles
        int64_t bq = 0;        // next position of the current batch
        int bn = 0;            // positions left in it
        int claim_raw = 0;     // lane 0: result of the claim in flight
        int claim_size = 0;    // its size; 0 = none in flight
        int size_hint = 1;
        int64_t last_q = blockIdx.x;  // last position handed out
        auto issue_claim = [&]() {
            if (lane == 0) claim_raw = atomicAdd(tile_counter, size_hint);
            claim_size = size_hint;
        };
        auto next_q = [&]() -> int64_t {
            if (!more) return mv.ntiles;
            if (bn == 0) {
                if (claim_size == 0) issue_claim();
                bq = int64_t(gridDim.x) + __shfl_sync(kFull, claim_raw, 0);
                bn = claim_size;
                claim_size = 0;
            }
            const int64_t q = bq++;
            --bn;
            last_q = q;
            if (q >= mv.ntiles) {
                more = false;
                return mv.ntiles;
            }
            if (bn == 0) issue_claim();  // the next batch, while this one is used
            return q;
        };
        fetch(blockIdx.x, ts[0], ms[0], rs[0]);
#pragma unroll
        for (int sl = 1; sl < kLook; ++sl) ts[sl] = kUnfetched;
        int i = 0;  // tiles published
        bool done = false;
        while (ok && !done) {
#pragma unroll
            for (int sl = 0; sl < kLook; ++sl) {
                if (done || !ok) break;
                if (ts[sl] == kUnfetched) fetch(next_q(), ts[sl], ms[sl], rs[sl]);
                // publish tile i for the MMA and epilogue roles
                const int r = i % kRing;
                if (!__all_sync(kFull, ptx::mbar_wait(&ring_empty[r], ((i / kRing) & 1) ^ 1, kWaitNs))) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (rs[sl][e] >= mv.n_out) rs[sl][e] = -1;  // only a malformed perm has such rows
                    ring[r].rows[e * 32 + lane] = rs[sl][e];
                }
                if (lane == 0) {
                    ring[r].tile = int32_t(ts[sl]);
                    ring[r].mask = ms[sl];
                }
                ptx::mbar_arrive(&ring_full[r]);
                ++i;
                if (ts[sl] < 0) {
                    ok = push_item(-1, rs[sl]);  // end of this CTA's items
                    done = true;
                    break;
                }
                for (uint32_t m = ms[sl]; m && ok; m &= m - 1) ok = push_item(__ffs(m) - 1, rs[sl]);
                {
                    const int64_t left = mv.ntiles - last_q, g = gridDim.x;
                    size_hint = __popc(ms[sl]) > 2 ? 1 : (left > 8 * g ? 4 : (left > 2 * g ? 2 : 1));
                }
                // refill: slots still unfetched come first (publish order), then this one
#pragma unroll
                for (int d = 1; d < kLook; ++d) {
                    const int o = (sl + d) % kLook;
                    if (ts[o] == kUnfetched) fetch(next_q(), ts[o], ms[o], rs[o]);
                }
                fetch(next_q(), ts[sl], ms[sl], rs[sl]);
            }
        }
        ptx::cp_async_wait<0>();
        if (!ok) s_abort = 1;
    }

    __syncthreads();
    if (s_abort) {
        // A role gave up: before the CTA releases its TMEM and shared memory,
        // everything still writing into them must land.  Every thread's
        // cp.async copies are complete (cp.async.wait_all above); thread 0
        // waits for the last weight-tile phase of each stage it filled (its TMA
        // bytes and the gather threads' arrivals), and the MMA thread commits
        // every MMA it issued to `drain` and waits for it.  These waits have
        // their own limit, independent of wait_ns.
        bad |= (tid == 0) ? LAT_ERR_TIMEOUT : 0;
        if (tid == 0) {
            for (uint32_t i = stages_issued > NS ? stages_issued - NS : 0; i < stages_issued; ++i)
                if (!ptx::mbar_wait(&full[i % NS], (i / NS) & 1, kDrainNs)) break;
        }
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

// ----------------------------------------------------------------------------- host side
using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

static EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

// Weights (k3, wrows, wcols) row-major viewed as a 2D (k3*wrows) x wcols tensor, 64 x 64 boxes, 128-byte swizzle.
static bool make_weight_map(CUtensorMap *map, const void *w, bool bf16, int k3, int wrows, int wcols) {
    EncodeFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(wcols), cuuint64_t(k3) * wrows};
    const cuuint64_t strides[1] = {cuuint64_t(wcols) * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void *>(w), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The weight tensor map of (w, shape, type), remembered per host thread for the
// last few weight tensors: encoding one is a driver call on every launch
// otherwise.  A map holds only the address, sizes and strides, so reusing it
// for the same (address, shape, type) is exact whatever the buffer holds.
static bool weight_map(CUtensorMap *map, const void *w, bool bf16, int k3, int wrows, int wcols) {
    struct Entry {
        const void *w = nullptr;
        int k3 = 0, rows = 0, cols = 0;
        bool bf16 = false;
        CUtensorMap map;
    };
    constexpr int kEntries = 8;
    thread_local Entry cache[kEntries];
    thread_local int next = 0;
    for (const Entry &e : cache)
        if (e.w == w && e.k3 == k3 && e.rows == wrows && e.cols == wcols && e.bf16 == bf16) {
            *map = e.map;
            return true;
        }
    if (!make_weight_map(map, w, bf16, k3, wrows, wcols)) return false;
    Entry &e = cache[next];
    next = (next + 1) % kEntries;
    e.w = w;
    e.k3 = k3;
    e.rows = wrows;
    e.cols = wcols;
    e.bf16 = bf16;
    e.map = *map;
    return true;
}

template <typename T, int KC, int N, bool BMN>
static lat_status launch(const void *x, const void *w, int k3, const MapView &mv, void *y, int32_t *counter,
                         int32_t *d_status, cudaStream_t s) {
    using C = Cfg<N>;
    CUtensorMap map;
    // forward: W[k] is (KC x N); data gradient: W[k] is (N x KC)
    if (!weight_map(&map, w, is_bf16<T>(), k3, BMN ? KC : N, BMN ? N : KC)) return LAT_ERR_CUDA;
    auto kern = conv_tc_kernel<T, KC, N, BMN>;
    const int64_t grid = std::min<int64_t>(mv.ntiles, GridCache<KernelTag<T, KC, N, BMN>>::get(kern, C::kSmem, int(C::kTmemCols), 2));
    if (grid <= 0) return LAT_ERR_CUDA;
    LAT_CUDA_TRY(fill_u32(counter, 1, 0u, s));
    LAT_CUDA_TRY(launch_pdl(kern, dim3(unsigned(grid)), dim3(kThreads), C::kSmem, s, map, static_cast<const T *>(x),
                            mv, static_cast<T *>(y), counter, wait_limit_ns(), d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

template <typename T, bool BMN>
static lat_status dispatch(int kc, int n, const void *x, const void *w, int k3, const MapView &mv, void *y,
                           int32_t *counter, int32_t *d_status, cudaStream_t s) {
    if (kc == 64 && n == 64) return launch<T, 64, 64, BMN>(x, w, k3, mv, y, counter, d_status, s);
    if (kc == 64 && n == 128) return launch<T, 64, 128, BMN>(x, w, k3, mv, y, counter, d_status, s);
    if (kc == 128 && n == 64) return launch<T, 128, 64, BMN>(x, w, k3, mv, y, counter, d_status, s);
    if (kc == 128 && n == 128) return launch<T, 128, 128, BMN>(x, w, k3, mv, y, counter, d_status, s);
    return LAT_ERR_UNSUPPORTED;
}

}  // namespace tc

bool conv_tc_supported(int kc, int n) { return (kc == 64 || kc == 128) && (n == 64 || n == 128); }

size_t conv_tc_ws_bytes() { return 256; }

// Forward (wt = false): gathered x (cin) x W[k] (cin x cout).  Data gradient (wt = true):
// gathered dy (kc = cout) x W[k]^T, producing n = cin channels.  ws: conv_tc_ws_bytes()
// bytes of scratch (the tile counter).
lat_status launch_conv_tc(bool bf16, const void *x, int kc, const void *w, int n, int k3, const MapView &mv, bool wt,
                          void *y, void *ws, int32_t *d_status, cudaStream_t s) {
    if (mv.ntiles == 0) return LAT_OK;
    int32_t *counter = static_cast<int32_t *>(ws);
    if (bf16)
        return wt ? tc::dispatch<__nv_bfloat16, false>(kc, n, x, w, k3, mv, y, counter, d_status, s)
                  : tc::dispatch<__nv_bfloat16, true>(kc, n, x, w, k3, mv, y, counter, d_status, s);
    return wt ? tc::dispatch<__half, false>(kc, n, x, w, k3, mv, y, counter, d_status, s)
              : tc::dispatch<__half, true>(kc, n, x, w, k3, mv, y, counter, d_status, s);
}

}  // namespace lat
