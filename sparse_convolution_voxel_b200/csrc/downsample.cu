// Output-support generation of a strided Conv3d (lat_downsample_ws_bytes,
// lat_downsample_coords).
//
// Torch Lattice docs, "Migrating from TorchSparse", "Convolution mapping":
// a strided forward convolution creates a downsampled support.  The coarse
// support is every q whose window {stride*q + off - pad, off in [0,K)^3}
// holds an active input.  Each input row proposes the coarse rows whose
// windows contain it (exactly one when K == stride and pad == 0: floor(p/s)).
// The proposals are made unique and put in canonical (b, x, y, z) order, so
// the result does not depend on the input row order.
//
// Two ways to sort + unique; one pass finds the range of every coarse field
// and the first is launched right behind it (its kernels read the range on
// the device), the second runs only when the first reports it did not apply:
//   * counting sort on a bitmap: when the fields, shifted to start at their
//     minimum, pack into a key of at most 30 bits and the bitmap is no larger
//     than max(2^24, 512 bits per proposal), every proposal sets its bit, a
//     scan of per-1024-bit popcounts gives each set bit its rank, and the
//     ranks are the sorted unique order;
//   * otherwise a radix sort of the packed 64-bit keys followed by unique.
// Both can also report each input's coarse row (its parent) when K == stride
// and pad == 0.
#include <cub/device/device_radix_sort.cuh>
#include <cub/device/device_select.cuh>

#include <climits>

#include "common.cuh"

namespace lat {

struct DownGeom {
    int ks[3], st[3], pd[3];
    int per_axis[3];  // candidate offsets per axis: ceil(K/s), or K when generating
    int cands;        // product of per_axis
    int up;           // 1: support of a generative transposed conv (every s*q + off - pad)
};

constexpr int kMaxBitmapBits = 30;

// Candidate coarse rows of every input as packed keys (EMPTY when a candidate
// does not exist), and the min / max of each coarse field over all candidates
// (range[0..3] = min b,x,y,z; range[4..7] = max).
__global__ void __launch_bounds__(256)
down_candidates_kernel(const int4 *__restrict__ coords, int64_t n, DownGeom g, uint64_t *__restrict__ keys,
                       int *__restrict__ range, int32_t *d_status) {
    pdl_enter();
    int mn[4] = {INT_MAX, INT_MAX, INT_MAX, INT_MAX}, mx[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
    const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (i < n) {
        const int4 c = __ldg(coords + i);
        uint64_t self;
        uint64_t *dst = keys + i * g.cands;
        if (!pack_key(c.x, c.y, c.z, c.w, self)) {
            for (int e = 0; e < g.cands; ++e) dst[e] = kEmptyKey;
            flag(d_status, LAT_ERR_COORD_RANGE);
        } else if (g.up) {
            // generated fine rows s*q + off - pad of coarse row q, off in [0,K)^3
            int e = 0;
            bool lost = false;
            for (int u = 0; u < g.ks[0]; ++u)
                for (int v = 0; v < g.ks[1]; ++v)
                    for (int w = 0; w < g.ks[2]; ++w, ++e) {
                        const int64_t f[3] = {int64_t(g.st[0]) * c.y + u - g.pd[0],
                                              int64_t(g.st[1]) * c.z + v - g.pd[1],
                                              int64_t(g.st[2]) * c.w + w - g.pd[2]};
                        uint64_t key = kEmptyKey;
                        const bool fits = f[0] >= -32768 && f[0] <= 32767 && f[1] >= -32768 && f[1] <= 32767 &&
                                          f[2] >= -32768 && f[2] <= 32767;
                        if (fits && pack_key(c.x, int(f[0]), int(f[1]), int(f[2]), key)) {
                            const int fv[4] = {c.x, int(f[0]), int(f[1]), int(f[2])};
#pragma unroll
                            for (int a = 0; a < 4; ++a) {
                                mn[a] = min(mn[a], fv[a]);
                                mx[a] = max(mx[a], fv[a]);
                            }
                        } else {
                            key = kEmptyKey;
                            lost = true;
                        }
                        dst[e] = key;
                    }
            if (lost) flag(d_status, LAT_ERR_COORD_RANGE);
        } else {
            const int p[3] = {c.y, c.z, c.w};
            int first[3];  // smallest off in [0,K) with (p - off + pad) divisible by s
#pragma unroll
            for (int a = 0; a < 3; ++a) first[a] = (p[a] + g.pd[a]) - floordiv(p[a] + g.pd[a], g.st[a]) * g.st[a];
            int e = 0;
            for (int u = 0; u < g.per_axis[0]; ++u)
                for (int v = 0; v < g.per_axis[1]; ++v)
                    for (int w = 0; w < g.per_axis[2]; ++w, ++e) {
                        const int off[3] = {first[0] + u * g.st[0], first[1] + v * g.st[1], first[2] + w * g.st[2]};
                        uint64_t key = kEmptyKey;
                        if (off[0] < g.ks[0] && off[1] < g.ks[1] && off[2] < g.ks[2]) {
                            int q[3];
#pragma unroll
                            for (int a = 0; a < 3; ++a) q[a] = (p[a] - off[a] + g.pd[a]) / g.st[a];  // exact
                            if (pack_key(c.x, q[0], q[1], q[2], key)) {
                                const int f[4] = {c.x, q[0], q[1], q[2]};
#pragma unroll
                                for (int a = 0; a < 4; ++a) {
                                    mn[a] = min(mn[a], f[a]);
                                    mx[a] = max(mx[a], f[a]);
                                }
                            } else {
                                key = kEmptyKey;
                            }
                        }
                        dst[e] = key;
                    }
        }
    }
    // warp, then block reduction: one set of global atomics per block (all blocks
    // update the same eight words, so per-warp atomics would serialise)
    __shared__ int s_mn[8][4], s_mx[8][4];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        for (int o = 16; o; o >>= 1) {
            mn[a] = min(mn[a], __shfl_xor_sync(0xFFFFFFFFu, mn[a], o));
            mx[a] = max(mx[a], __shfl_xor_sync(0xFFFFFFFFu, mx[a], o));
        }
        if (lane == 0) {
            s_mn[warp][a] = mn[a];
            s_mx[warp][a] = mx[a];
        }
    }
    __syncthreads();
    if (threadIdx.x < 4) {
        const int a = threadIdx.x;
        int bmn = INT_MAX, bmx = INT_MIN;
        for (int w = 0; w < int(blockDim.x >> 5); ++w) {
            bmn = min(bmn, s_mn[w][a]);
            bmx = max(bmx, s_mx[w][a]);
        }
        if (bmn != INT_MAX) {
            atomicMin(range + a, bmn);
            atomicMax(range + 4 + a, bmx);
        }
    }
}

// range[0..3] = INT_MAX, range[4..7] = INT_MIN (the candidates pass reduces into
// them), range[8] = 0 (the count pass's arrival counter).
__global__ void range_init_kernel(int *range) {
    pdl_enter();
    if (threadIdx.x < 4) range[threadIdx.x] = INT_MAX;
    else if (threadIdx.x < 8) range[threadIdx.x] = INT_MIN;
    else if (threadIdx.x == 8) range[8] = 0;
}

// Order-preserving compact key of a coarse row: fields shifted to their minimum, packed.
struct Compact {
    int mn[4];
    int w[4];  // bit widths of b, x, y, z
    __device__ __forceinline__ uint32_t pack(uint64_t key) const {
        int4 c;
        unpack_key(key, c);
        uint32_t v = uint32_t(c.x - mn[0]);
        v = (v << w[1]) | uint32_t(c.y - mn[1]);
        v = (v << w[2]) | uint32_t(c.z - mn[2]);
        v = (v << w[3]) | uint32_t(c.w - mn[3]);
        return v;
    }
    __device__ __forceinline__ int4 unpack(uint32_t v) const {
        int4 c;
        c.w = int(v & ((1u << w[3]) - 1u)) + mn[3];
        v >>= w[3];
        c.z = int(v & ((1u << w[2]) - 1u)) + mn[2];
        v >>= w[2];
        c.y = int(v & ((1u << w[1]) - 1u)) + mn[1];
        v >>= w[1];
        c.x = int(v) + mn[0];
        return c;
    }
};

// Bitmap plan from the device-side field ranges: the compact layout, the
// group count (1024 bits per group), whether the bitmap path applies (ok) and
// whether there is no coarse row at all (empty).  Every bitmap kernel derives
// it itself, so the host does not wait for the range pass.
struct Plan {
    Compact cp;
    int64_t ngroups;
    bool ok, empty;
};
__device__ __forceinline__ Plan make_plan(const int *__restrict__ range, int64_t budget_bits) {
    Plan p;
    p.empty = __ldg(range) == INT_MAX;
    int total = 0;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int lo = __ldg(range + a), hi = __ldg(range + 4 + a);
        const int64_t span = p.empty ? 0 : int64_t(hi) - lo;
        p.cp.mn[a] = lo;
        p.cp.w[a] = span > 0 ? 64 - __clzll(span) : 0;
        total += p.cp.w[a];
    }
    p.ok = !p.empty && total <= kMaxBitmapBits && (int64_t(1) << total) <= budget_bits;
    p.ngroups = p.ok ? max(int64_t(1), (int64_t(1) << total) / 1024) : 0;
    return p;
}

__global__ void __launch_bounds__(256)
bitmap_zero_kernel(const int *__restrict__ range, int64_t budget_bits, uint4 *__restrict__ bitmap) {
    pdl_enter();
    const Plan p = make_plan(range, budget_bits);
    const int64_t n4 = p.ngroups * 8;  // 32 words per group
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n4; e += int64_t(gridDim.x) * blockDim.x)
        bitmap[e] = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(256)
bitmap_mark_kernel(const uint64_t *__restrict__ keys, int64_t items, const int *__restrict__ range,
                   int64_t budget_bits, uint32_t *__restrict__ bitmap) {
    pdl_enter();
    const int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (e >= items) return;
    const Plan p = make_plan(range, budget_bits);
    if (!p.ok) return;
    const uint64_t key = keys[e];
    if (key == kEmptyKey) return;
    const uint32_t v = p.cp.pack(key);
    atomicOr(bitmap + (v >> 5), 1u << (v & 31));
}

// Set bits per group of 32 words (1024 bits): grp_cnt, and grp_pre = the
// exclusive prefix of grp_cnt within each block of 256 groups; blk_cnt = the
// block's total.  The last block to finish (an arrival counter that the range
// pass zeroes) scans blk_cnt into blk_off and writes the coarse row count, or
// -1 when the bitmap path does not apply (0 when there is no row at all), so
// no separate scan launch is needed.  Blocks past the plan's groups only
// return; the arrival count is over the blocks that cover groups.
__global__ void __launch_bounds__(256)
bitmap_count_kernel(const uint32_t *__restrict__ bitmap, int *__restrict__ range, int64_t budget_bits,
                    int32_t *__restrict__ grp_cnt, int32_t *__restrict__ grp_pre, int32_t *__restrict__ blk_cnt,
                    int64_t *__restrict__ blk_off, int64_t *__restrict__ n_out_dev) {
    pdl_enter();
    __shared__ int s_warp[8];
    __shared__ int64_t s_big[8];
    __shared__ bool s_last;
    const Plan p = make_plan(range, budget_bits);
    const int64_t nblk = (p.ngroups + 255) / 256;
    if (nblk == 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) *n_out_dev = p.empty ? 0 : -1;
        return;
    }
    if (int64_t(blockIdx.x) >= nblk) return;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t gi = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    int c = 0;
    if (gi < p.ngroups) {
        const uint4 *w4 = reinterpret_cast<const uint4 *>(bitmap + gi * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint4 v = __ldg(w4 + e);
            c += __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
        }
    }
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
    }
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    int before = 0;
    for (int q = 0; q < w; ++q) before += s_warp[q];
    if (gi < p.ngroups) {
        grp_cnt[gi] = c;
        grp_pre[gi] = before + incl - c;
    }
    if (threadIdx.x == 0) {
        int t = 0;
        for (int q = 0; q < 8; ++q) t += s_warp[q];
        blk_cnt[blockIdx.x] = t;
        __threadfence();
        s_last = atomicAdd(range + 8, 1) == int(nblk - 1);
    }
    __syncthreads();
    if (!s_last) return;
    // last block: exclusive scan of the block totals (each thread a run of them)
    __threadfence();
    const int64_t per = (nblk + 255) / 256;
    const int64_t b0 = min(nblk, threadIdx.x * per), b1 = min(nblk, b0 + per);
    int64_t sum = 0;
    for (int64_t i = b0; i < b1; ++i) sum += __ldcg(blk_cnt + i);
    int64_t inc = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int64_t o = __shfl_up_sync(0xFFFFFFFFu, inc, d);
        if (lane >= d) inc += o;
    }
    if (lane == 31) s_big[w] = inc;
    __syncthreads();
    int64_t run = inc - sum;
    for (int q = 0; q < w; ++q) run += s_big[q];
    for (int64_t i = b0; i < b1; ++i) {
        blk_off[i] = run;
        run += __ldcg(blk_cnt + i);
    }
    if (threadIdx.x == 255) *n_out_dev = run;
}

// Two roles in one launch, both reading only the count pass's results:
//   blocks [0, emit_blocks): warps walk the 1024-bit groups (grid-stride, 32
//     groups at a time, skipping empty ones); per group each lane takes one word: a warp scan of the word popcounts gives every set bit its
//     rank = blk_off + grp_pre + the bits before it, and the lane writes the
//     coordinates of its bits (bit order = canonical order);
//   the remaining blocks: one thread per input, its (single) proposal's rank
//     among the set bits = its coarse row (parent); -1 for an input without
//     one.  Nothing is written when the bitmap path does not apply.
__global__ void __launch_bounds__(256)
bitmap_emit_kernel(const uint32_t *__restrict__ bitmap, const int *__restrict__ range, int64_t budget_bits,
                   const int32_t *__restrict__ grp_cnt, const int32_t *__restrict__ grp_pre,
                   const int64_t *__restrict__ blk_off, int4 *__restrict__ out, int64_t capacity, int emit_blocks,
                   const uint64_t *__restrict__ keys, int64_t n_in, int32_t *__restrict__ parent) {
    pdl_enter();
    const Plan p = make_plan(range, budget_bits);
    if (!p.ok) return;
    const int lane = threadIdx.x & 31;
    if (int(blockIdx.x) < emit_blocks) {
        // a warp takes 32 consecutive groups at a time: one coalesced load of their
        // counts, then only the non-empty ones (most groups of a sparse bitmap are empty)
        const int64_t nwarps = int64_t(emit_blocks) * (blockDim.x >> 5);
        const int64_t nchunks = (p.ngroups + 31) / 32;
        for (int64_t ch = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); ch < nchunks; ch += nwarps) {
            const int64_t gl = ch * 32 + lane;
            unsigned busy = __ballot_sync(0xFFFFFFFFu, gl < p.ngroups && __ldg(grp_cnt + gl) != 0);
            while (busy) {
                const int64_t g = ch * 32 + __ffs(busy) - 1;
                busy &= busy - 1;
                uint32_t word = __ldg(bitmap + g * 32 + lane);
                const int pc = __popc(word);
                int incl = pc;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                    if (lane >= d) incl += o;
                }
                int64_t rank = __ldg(blk_off + (g >> 8)) + __ldg(grp_pre + g) + incl - pc;
                while (word) {
                    const int b = __ffs(word) - 1;
                    word &= word - 1;
                    if (rank < capacity) out[rank] = p.cp.unpack(uint32_t(g * 1024 + lane * 32 + b));
                    ++rank;
                }
            }
        }
        return;
    }
    const int64_t i = (int64_t(blockIdx.x) - emit_blocks) * blockDim.x + threadIdx.x;
    if (i >= n_in) return;
    const uint64_t key = keys[i];
    if (key == kEmptyKey) {
        parent[i] = -1;
        return;
    }
    const uint32_t v = p.cp.pack(key);
    const uint32_t gi = v >> 10, wi = (v >> 5) & 31;
    // bits of the group before v: whole words below wi, then the low bits of word wi
    const uint32_t *gw = bitmap + int64_t(gi) * 32;
    int64_t rank = __ldg(blk_off + (gi >> 8)) + __ldg(grp_pre + gi);
    for (uint32_t e = 0; e < (wi & ~3u); e += 4) {
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(gw + e));
        rank += __popc(q.x) + __popc(q.y) + __popc(q.z) + __popc(q.w);
    }
    for (uint32_t e = wi & ~3u; e < wi; ++e) rank += __popc(__ldg(gw + e));
    rank += __popc(__ldg(gw + wi) & ((1u << (v & 31)) - 1u));
    parent[i] = int32_t(rank);
}

// Unpack the unique keys (the last one may be the EMPTY filler) into coordinate rows.
__global__ void __launch_bounds__(256)
down_unpack_kernel(const uint64_t *__restrict__ uniq, const int *__restrict__ n_uniq, int4 *__restrict__ out,
                   int64_t capacity, int64_t *__restrict__ n_out_dev) {
    pdl_enter();
    const int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    int64_t m = *n_uniq;
    if (m > 0 && uniq[m - 1] == kEmptyKey) --m;
    if (r == 0) *n_out_dev = m;
    if (r >= m || r >= capacity) return;
    int4 c;
    unpack_key(uniq[r], c);
    out[r] = c;
}

// Coarse row of each input by binary search in the sorted unique keys.
__global__ void __launch_bounds__(256)
sorted_parent_kernel(const uint64_t *__restrict__ keys, int64_t n, const uint64_t *__restrict__ uniq,
                     const int64_t *__restrict__ n_out_dev, int32_t *__restrict__ parent) {
    pdl_enter();
    const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (i >= n) return;
    const uint64_t key = keys[i];
    int64_t lo = 0, hi = *n_out_dev;
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (uniq[mid] < key) lo = mid + 1;
        else hi = mid;
    }
    parent[i] = (key != kEmptyKey && lo < *n_out_dev && uniq[lo] == key) ? int32_t(lo) : -1;
}

// up = false: the support of a strided / generative Conv3d (geom->mode LAT_STRIDED);
// up = true: the support a GenerativeConvTranspose3d generates (LAT_TRANSPOSED).
static bool down_geom(const lat_geom *geom, DownGeom &g, bool up = false) {
    if (!geom || geom->mode != (up ? LAT_TRANSPOSED : LAT_STRIDED)) return false;
    g.up = up ? 1 : 0;
    g.cands = 1;
    for (int a = 0; a < 3; ++a) {
        if (geom->ksize[a] < 1 || geom->stride[a] < 1 || geom->pad[a] < 0 || geom->pad[a] >= geom->ksize[a] + 32768)
            return false;
        g.ks[a] = geom->ksize[a];
        g.st[a] = geom->stride[a];
        g.pd[a] = geom->pad[a];
        g.per_axis[a] = up ? geom->ksize[a] : (geom->ksize[a] + geom->stride[a] - 1) / geom->stride[a];
        g.cands *= g.per_axis[a];
    }
    return g.ks[0] * g.ks[1] * g.ks[2] <= 32;
}

// Largest bitmap (bits) the counting-sort path may use for `items` proposals.
static int64_t bitmap_budget_bits(int64_t items) {
    int64_t b = std::max<int64_t>(int64_t(1) << 24, 512 * items);
    return std::min<int64_t>(b, int64_t(1) << kMaxBitmapBits);
}

struct DownWs {
    uint64_t *keys;
    int *range;
    int64_t *n_out_dev;
    // sort path
    uint64_t *sorted, *uniq;
    int *n_uniq;
    void *sort_tmp, *sel_tmp;
    size_t sort_bytes, sel_bytes;
    // bitmap path
    uint32_t *bitmap;
    int32_t *grp_cnt;
    int32_t *grp_pre;
    int32_t *blk_cnt;
    int64_t *blk_off;
    int64_t max_groups;
    size_t total;
};

static DownWs carve_down_ws(void *base, int64_t items) {
    DownWs w{};
    Carver cv(base);
    w.keys = cv.take<uint64_t>(size_t(items));
    w.range = cv.take<int>(16);
    w.n_out_dev = cv.take<int64_t>(1);
    const size_t common = cv.used;
    // sort path
    w.sorted = cv.take<uint64_t>(size_t(items));
    w.uniq = cv.take<uint64_t>(size_t(items));
    w.n_uniq = cv.take<int>(1);
    cub::DeviceRadixSort::SortKeys(nullptr, w.sort_bytes, (const uint64_t *)nullptr, (uint64_t *)nullptr,
                                   int(items), 0, 64);
    cub::DeviceSelect::Unique(nullptr, w.sel_bytes, (const uint64_t *)nullptr, (uint64_t *)nullptr, (int *)nullptr,
                              int(items));
    w.sort_tmp = cv.take<char>(w.sort_bytes);
    w.sel_tmp = cv.take<char>(w.sel_bytes);
    const size_t sort_end = cv.used;
    // bitmap path (overlaps the sort path's buffers)
    cv.used = common;
    const int64_t bits = bitmap_budget_bits(items);
    w.max_groups = std::max<int64_t>(1, bits / 1024);
    w.bitmap = cv.take<uint32_t>(size_t(w.max_groups) * 32);
    w.grp_cnt = cv.take<int32_t>(size_t(w.max_groups));
    w.grp_pre = cv.take<int32_t>(size_t(w.max_groups));
    const int64_t max_blk = (w.max_groups + 255) / 256;
    w.blk_cnt = cv.take<int32_t>(size_t(max_blk));
    w.blk_off = cv.take<int64_t>(size_t(max_blk));
    w.total = align_up(std::max(sort_end, cv.used), 256);
    return w;
}

}  // namespace lat

extern "C" size_t lat_downsample_ws_bytes(int64_t n_in, const lat_geom *geom) {
    lat::DownGeom g;
    if (n_in < 0 || !lat::down_geom(geom, g)) return 0;
    const int64_t items = n_in * g.cands;
    if (items >= (int64_t(1) << 31)) return 0;
    return lat::carve_down_ws(nullptr, std::max<int64_t>(items, 1)).total;
}

namespace lat {

// Checks shared by both entry points; fills g, w, items.  LAT_OK with items == 0
// means there is nothing to do (no input row).
static lat_status down_prepare(const int32_t *coords, int64_t n_in, const lat_geom *geom, int32_t *out_coords,
                               int64_t out_capacity, int32_t *parent, void *ws, size_t ws_bytes, DownGeom &g,
                               DownWs &w, int64_t &items, bool up = false) {
    items = 0;
    if (n_in < 0 || out_capacity < 0 || !down_geom(geom, g, up)) return LAT_ERR_ARG;
    if (n_in > 0 && (!coords || (out_capacity > 0 && !out_coords))) return LAT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(coords) % 16 || reinterpret_cast<uintptr_t>(out_coords) % 16) return LAT_ERR_ARG;
    if (parent) {  // one coarse row per input only when the kernel tiles the stride exactly
        for (int a = 0; a < 3; ++a)
            if (g.ks[a] != g.st[a] || g.pd[a] != 0) return LAT_ERR_UNSUPPORTED;
    }
    const int64_t n_items = n_in * g.cands;
    if (n_items >= (int64_t(1) << 31)) return LAT_ERR_UNSUPPORTED;
    if (n_in == 0) return LAT_OK;
    const DownWs need = carve_down_ws(nullptr, n_items);
    if (!ws || ws_bytes < need.total) return LAT_ERR_WORKSPACE;
    w = carve_down_ws(ws, n_items);
    items = n_items;
    return LAT_OK;
}

// Range pass and the bitmap counting-sort path, launched without waiting for
// the range: every kernel derives the plan on the device, grids cover the
// largest bitmap the budget allows, and w.n_out_dev ends up holding the coarse
// row count, or -1 when the path did not apply.
static lat_status enqueue_bitmap_path(const int32_t *coords, int64_t n_in, const DownGeom &g, int64_t items,
                                      int32_t *out_coords, int64_t out_capacity, int32_t *parent, const DownWs &w,
                                      int32_t *d_status, cudaStream_t s) {
    const unsigned in_blocks = unsigned((n_in + 255) / 256), item_blocks = unsigned((items + 255) / 256);
    LAT_CUDA_TRY(launch_pdl(range_init_kernel, dim3(1), dim3(32), 0, s, w.range));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(down_candidates_kernel, dim3(in_blocks), dim3(256), 0, s,
                            reinterpret_cast<const int4 *>(coords), n_in, g, w.keys, w.range, d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    const int64_t budget = bitmap_budget_bits(items);
    const unsigned gblocks = unsigned((w.max_groups + 255) / 256);
    const unsigned zblocks = unsigned(std::min<int64_t>((w.max_groups * 8 + 255) / 256, int64_t(num_sms()) * 8));
    LAT_CUDA_TRY(launch_pdl(bitmap_zero_kernel, dim3(zblocks), dim3(256), 0, s, w.range, budget,
                            reinterpret_cast<uint4 *>(w.bitmap)));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(bitmap_mark_kernel, dim3(item_blocks), dim3(256), 0, s, w.keys, items, w.range, budget,
                            w.bitmap));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(bitmap_count_kernel, dim3(gblocks), dim3(256), 0, s, w.bitmap, w.range, budget, w.grp_cnt,
                            w.grp_pre, w.blk_cnt, w.blk_off, w.n_out_dev));
    LAT_CUDA_TRY(cudaGetLastError());
    const int emit_blocks = int(std::min<int64_t>((w.max_groups + 255) / 256, int64_t(num_sms()) * 8));
    const unsigned parent_blocks = parent ? in_blocks : 0u;
    LAT_CUDA_TRY(launch_pdl(bitmap_emit_kernel, dim3(unsigned(emit_blocks) + parent_blocks), dim3(256), 0, s, w.bitmap,
                            w.range, budget, w.grp_cnt, w.grp_pre, w.blk_off, reinterpret_cast<int4 *>(out_coords),
                            out_capacity, emit_blocks, w.keys, parent ? n_in : int64_t(0), parent));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

}  // namespace lat

namespace lat {
static lat_status support_blocking(const int32_t *coords, int64_t n_in, const lat_geom *geom, int32_t *out_coords,
                                   int64_t out_capacity, int64_t *n_out, int32_t *parent, void *ws, size_t ws_bytes,
                                   int32_t *d_status, lat_stream stream, bool up) {
    if (!n_out) return LAT_ERR_ARG;
    DownGeom g;
    DownWs w;
    int64_t items = 0;
    const lat_status st =
        down_prepare(coords, n_in, geom, out_coords, out_capacity, parent, ws, ws_bytes, g, w, items, up);
    if (st != LAT_OK) return st;
    *n_out = 0;
    if (items == 0) return LAT_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned in_blocks = unsigned((n_in + 255) / 256), item_blocks = unsigned((items + 255) / 256);
    const lat_status eq = enqueue_bitmap_path(coords, n_in, g, items, out_coords, out_capacity, parent, w, d_status, s);
    if (eq != LAT_OK) return eq;
    int64_t m = 0;
    LAT_CUDA_TRY(cudaMemcpyAsync(&m, w.n_out_dev, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    LAT_CUDA_TRY(cudaStreamSynchronize(s));
    if (m < 0) {
        // ------------------------------------------------ radix sort + unique of the packed keys
        size_t b = w.sort_bytes;
        LAT_CUDA_TRY(cub::DeviceRadixSort::SortKeys(w.sort_tmp, b, w.keys, w.sorted, int(items), 0, 64, s));
        b = w.sel_bytes;
        LAT_CUDA_TRY(cub::DeviceSelect::Unique(w.sel_tmp, b, w.sorted, w.uniq, w.n_uniq, int(items), s));
        LAT_CUDA_TRY(launch_pdl(down_unpack_kernel, dim3(item_blocks), dim3(256), 0, s, w.uniq, w.n_uniq,
                                reinterpret_cast<int4 *>(out_coords), out_capacity, w.n_out_dev));
        LAT_CUDA_TRY(cudaGetLastError());
        if (parent) {
            LAT_CUDA_TRY(launch_pdl(sorted_parent_kernel, dim3(in_blocks), dim3(256), 0, s, w.keys, n_in, w.uniq,
                                    w.n_out_dev, parent));
            LAT_CUDA_TRY(cudaGetLastError());
        }
        LAT_CUDA_TRY(cudaMemcpyAsync(&m, w.n_out_dev, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
        LAT_CUDA_TRY(cudaStreamSynchronize(s));
    }
    *n_out = m;
    return m > out_capacity ? LAT_ERR_CAPACITY : LAT_OK;
}
}  // namespace lat

extern "C" lat_status lat_downsample_coords(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                                            int32_t *out_coords, int64_t out_capacity, int64_t *n_out,
                                            int32_t *parent, void *ws, size_t ws_bytes, int32_t *d_status,
                                            lat_stream stream) {
    return lat::support_blocking(coords, n_in, geom, out_coords, out_capacity, n_out, parent, ws, ws_bytes, d_status,
                                 stream, false);
}

extern "C" size_t lat_upsample_ws_bytes(int64_t n_in, const lat_geom *geom) {
    lat::DownGeom g;
    if (n_in < 0 || !lat::down_geom(geom, g, true)) return 0;
    const int64_t items = n_in * g.cands;
    if (items >= (int64_t(1) << 31)) return 0;
    return lat::carve_down_ws(nullptr, std::max<int64_t>(items, 1)).total;
}

extern "C" lat_status lat_upsample_coords(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                                          int32_t *out_coords, int64_t out_capacity, int64_t *n_out, void *ws,
                                          size_t ws_bytes, int32_t *d_status, lat_stream stream) {
    return lat::support_blocking(coords, n_in, geom, out_coords, out_capacity, n_out, nullptr, ws, ws_bytes,
                                 d_status, stream, true);
}

extern "C" lat_status lat_downsample_coords_async(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                                                  int32_t *out_coords, int64_t out_capacity, int64_t *n_out_host,
                                                  int32_t *parent, void *ws, size_t ws_bytes, int32_t *d_status,
                                                  lat_stream stream) {
    using namespace lat;
    if (!n_out_host) return LAT_ERR_ARG;
    DownGeom g;
    DownWs w;
    int64_t items = 0;
    const lat_status st = down_prepare(coords, n_in, geom, out_coords, out_capacity, parent, ws, ws_bytes, g, w, items);
    if (st != LAT_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (items == 0) {
        *n_out_host = 0;
        return LAT_OK;
    }
    const lat_status eq = enqueue_bitmap_path(coords, n_in, g, items, out_coords, out_capacity, parent, w, d_status, s);
    if (eq != LAT_OK) return eq;
    LAT_CUDA_TRY(cudaMemcpyAsync(n_out_host, w.n_out_dev, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    return LAT_OK;
}
