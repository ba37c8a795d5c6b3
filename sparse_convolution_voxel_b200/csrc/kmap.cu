// Kernel-map construction / coordinate query (lat_kmap_ws_bytes, lat_kmap_query).
//
// Torch Lattice docs, "Migrating from TorchSparse": kernel-map construction
// and coordinate query are CUDA kernels of the library ("What remains
// familiar", "Sparse tensor expectations"), and the support semantics come
// from the "Convolution mapping" table.  Pipeline (all on `stream`):
//   1. probe:  strided / transposed maps: one thread per output row probes
//              every offset and writes nbr (offset-major, coalesced), mask and
//              per (offset, block) hit counts from warp ballots.  Submanifold
//              maps: one thread per (row, offset below the centre), each hit
//              mirrored (the relation is symmetric) and ORed into both masks
//              atomically; a count pass over the masks gives the counts.
//   2. scan:   one block per offset turns its per-block counts into offsets
//              (pairs come out grouped by offset, rows ascending).
//   3. emit:   walks the masks and writes (in, out) pairs at ballot-ranked
//              positions, reading nbr only where a bit is set:
//              deterministic, no atomics.
//   4. sort:   stable LSD radix sort (8-bit digits: 2 passes for the 16-bit
//              grouping key of the mask -- neighbour count, mask hash --, 1
//              pass when k3 <= 8) of the output rows -> perm; the last pass
//              ORs the masks of each LAT_TILE_ROWS run of perm -> tile_mask.
#include "common.cuh"

namespace lat {

constexpr int kQueryThreads = 256;
constexpr int kQueryWarps = kQueryThreads / 32;

struct Geom {
    int ks[3], st[3], pd[3];
    int mode;
    int k3;
    signed char off[32][3];  // (ix, iy, iz) of offset k
    // Unit stride on every axis: the probed coordinate is the row's own plus a
    // fixed vector, so the probed key is the row's key plus a packed delta as long
    // as no field leaves [0, 65535] (row coordinates within [lo, hi] per axis).
    int shift;
    long long delta[32];
    int lo[3], hi[3];
};

constexpr int kProbeBatch = 8;  // slot loads a thread keeps in flight
constexpr int kGroupKeyBits = 16;

// Sort key that groups output rows for the convolution tiles: the number of
// neighbours (capped at 31) in the top 5 bits, then 11 bits of a multiplicative
// hash of the mask.  Rows with equal masks share a key; sorting by it keeps the
// union of masks inside a 128-row tile as small as an exact sort by mask does
// on the LiDAR- and image-shaped inputs, in 2 radix passes instead of 4.
// With at most 8 offsets the mask itself is the key (exact, one radix pass).
__device__ __forceinline__ uint32_t group_key(uint32_t m, int k3) {
    if (k3 <= 8) return m;
    const uint32_t pc = min(__popc(m), 31);
    return (pc << 11) | ((m * 0x9E3779B1u) >> 21);
}
inline int group_key_bits(int k3) { return k3 <= 8 ? k3 : kGroupKeyBits; }

// ----------------------------------------------------------------------------- row sort
// Stable LSD radix sort of the row grouping keys (8-bit digits, one pass per
// digit) producing perm.  The input of a pass is cut into tiles of kSortTile
// rows; hist[d * ntile + b] counts digit d in tile b.  The first pass's
// histogram is accumulated by the kernel that computes the keys
// (sort_hist_add), each pass's scatter accumulates the next pass's histogram;
// one block per digit scans that digit's per-tile counts, and every scatter
// block scans the 256 digit totals, which together give the first output
// position of every (digit, tile).  Within a tile, rows keep their order (ranks from warp
// match + per-warp digit counts), so the result is the stable sort: perm equals
// the stable argsort of the keys, deterministic.  The last pass also ORs every
// row's mask into its tile of LAT_TILE_ROWS output positions.
constexpr int kSortThreads = 256;
constexpr int kSortRounds = 2;
constexpr int kSortTile = kSortThreads * kSortRounds;
static_assert(kSortTile >= 512, "next-pass tag packs the output tile in 22 bits");
constexpr int kSortWarps = kSortThreads / 32;

// Adds the lowest digit of this lane's key to the first pass's histogram.  Every
// lane of the warp calls it; the warp's rows lie in one sort tile.
__device__ __forceinline__ void sort_hist_add(uint32_t key, bool live, int64_t j, int32_t *__restrict__ hist,
                                              int ntile) {
    const int lane = threadIdx.x & 31;
    const uint32_t d = key & 255u;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d : 256u + lane);
    if (live && (peers & ((1u << lane) - 1u)) == 0)
        atomicAdd(hist + int64_t(d) * ntile + j / kSortTile, int(__popc(peers)));
}

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

// One thread per output row.  Offsets are probed in batches of kProbeBatch:
// each round loads the 4 keys of the current slot group of every unresolved
// offset of the batch at once (two 16-byte loads per group), then resolves
// what it can (a match, or an empty slot before it, ends the probe); the rows
// of the matches are loaded together after the rounds.  At the table's load
// factor nearly every probe ends inside its home group, so a batch takes about
// one round.  Rounds are bounded by the probe window (kMaxProbeSlots).  Strided and transposed
// maps (submanifold maps use kmap_probe_sym_kernel): every offset is probed and
// the mask, grouping key, first sort histogram and per-block counts are
// produced here.
__global__ void __launch_bounds__(kQueryThreads)
kmap_probe_kernel(const SlotGroup *__restrict__ groups, uint32_t cap_mask, const int4 *__restrict__ out_coords,
                  int64_t n_out, int64_t n_in, Geom g, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask,
                  uint32_t *__restrict__ keys, int32_t *__restrict__ hist, int ntile, int32_t *__restrict__ block_counts,
                  int nblk, int32_t *d_status) {
    pdl_enter();
    __shared__ int s_cnt[32];
    if (threadIdx.x < 32) s_cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const bool live = j < n_out;
    int4 c = make_int4(0, 0, 0, 0);
    if (live) c = __ldg(out_coords + j);
    const int kend = g.k3;
    uint64_t self = 0;
    const bool fast = live && g.shift && c.y >= g.lo[0] && c.y <= g.hi[0] && c.z >= g.lo[1] && c.z <= g.hi[1] &&
                      c.w >= g.lo[2] && c.w <= g.hi[2] && pack_key(c.x, c.y, c.z, c.w, self);
    uint32_t m = 0;
    int32_t bad = 0;
    for (int k0 = 0; k0 < kend; k0 += kProbeBatch) {
        uint64_t key[kProbeBatch];
        uint32_t slot[kProbeBatch];  // first slot of the group probed next
        int hit[kProbeBatch];        // slot of the match, -1 = none
        int row[kProbeBatch];
        uint32_t pending = 0;
#pragma unroll
        for (int e = 0; e < kProbeBatch; ++e) {
            const int k = k0 + e;
            row[e] = -1;
            hit[e] = -1;
            key[e] = kEmptyKey;
            slot[e] = 0;
            if (!live || k >= kend) continue;
            bool ok;
            if (fast) {
                key[e] = self + uint64_t(g.delta[k]);
                ok = true;
            } else {
                ok = query_coord(g, c, g.off[k][0], g.off[k][1], g.off[k][2], key[e]);
            }
            if (ok) {
                slot[e] = probe_start(key[e], cap_mask);
                pending |= 1u << e;
            }
        }
        for (uint32_t round = 0; pending && round < probe_window(cap_mask) / kGroupSlots; ++round) {
            ulonglong2 ka[kProbeBatch], kb[kProbeBatch];
#pragma unroll
            for (int e = 0; e < kProbeBatch; ++e) {
                if (pending & (1u << e)) {
                    const SlotGroup *gp = groups + slot[e] / kGroupSlots;
                    ka[e] = __ldg(reinterpret_cast<const ulonglong2 *>(gp->key));
                    kb[e] = __ldg(reinterpret_cast<const ulonglong2 *>(gp->key + 2));
                }
            }
#pragma unroll
            for (int e = 0; e < kProbeBatch; ++e) {
                if (!(pending & (1u << e))) continue;
                const uint64_t k4[kGroupSlots] = {ka[e].x, ka[e].y, kb[e].x, kb[e].y};
                int found = -1;
                bool stop = false;
#pragma unroll
                for (int i = 0; i < kGroupSlots; ++i) {
                    if (stop) continue;
                    if (k4[i] == key[e]) {
                        found = i;
                        stop = true;
                    } else if (k4[i] == kEmptyKey) {
                        stop = true;
                    }
                }
                if (stop) {
                    pending &= ~(1u << e);
                    if (found >= 0) hit[e] = int(slot[e]) + found;
                } else {
                    slot[e] = (slot[e] + kGroupSlots) & cap_mask;
                }
            }
        }
#pragma unroll
        for (int e = 0; e < kProbeBatch; ++e)
            if (hit[e] >= 0) row[e] = int(__ldg(&groups[hit[e] / kGroupSlots].row[hit[e] % kGroupSlots]));
#pragma unroll
        for (int e = 0; e < kProbeBatch; ++e) {
            const int k = k0 + e;
            if (k >= kend) break;
            int r = row[e];
            if (r >= n_in) { bad |= LAT_ERR_BAD_MAP; r = -1; }
            if (live) nbr[int64_t(k) * n_out + j] = r;
            const unsigned hits = __ballot_sync(0xFFFFFFFFu, r >= 0);
            if (r >= 0) m |= 1u << k;
            if ((threadIdx.x & 31) == 0 && hits) atomicAdd(&s_cnt[k], __popc(hits));
        }
    }
    if (bad) flag(d_status, bad);
    const uint32_t key = group_key(m, g.k3);
    if (live) {
        mask[j] = m;
        keys[j] = key;
    }
    sort_hist_add(key, live, j, hist, ntile);
    __syncthreads();
    if (threadIdx.x < g.k3) block_counts[int64_t(threadIdx.x) * nblk + blockIdx.x] = s_cnt[threadIdx.x];
}

// Submanifold map, step 0: the centre row of nbr (every row is its own centre
// neighbour), -1 in every offset above the centre (filled by mirrored hits
// only), masks holding just the centre bit, and zeroed sort histograms and
// tile masks.  One thread per row; all stores coalesced.
__global__ void __launch_bounds__(kQueryThreads)
kmap_subm_init_kernel(int64_t n_out, int k3, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask,
                      int32_t *__restrict__ hist, int64_t hist_words, uint32_t *__restrict__ tile_mask,
                      int64_t ntiles) {
    pdl_enter();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    // the row sort's digit histograms and the tile masks start at zero
    const int64_t stride = int64_t(gridDim.x) * kQueryThreads;
    for (int64_t i = j; i < hist_words; i += stride) hist[i] = 0;
    for (int64_t i = j; i < ntiles; i += stride) tile_mask[i] = 0;
    if (j >= n_out) return;
    const int centre = k3 / 2;
    nbr[int64_t(centre) * n_out + j] = int32_t(j);
    for (int k = centre + 1; k < k3; ++k) nbr[int64_t(k) * n_out + j] = -1;
    mask[j] = 1u << centre;
}

// Submanifold map, step 1: one thread per (offset k below the centre, row j);
// blockIdx.y is the offset, so a warp probes one offset for 32 consecutive rows
// (coalesced coordinate loads and nbr stores, a uniform key delta).  A probe
// reads its home group's 4 keys with two 16-byte loads and walks on to the next
// group only when all 4 slots hold other keys (bounded by the probe window).
// A hit at row r also writes the mirrored entry nbr[k3-1-k][r] = j (the
// relation is symmetric) and ORs both bits into the masks.  Far fewer
// instructions per lookup than looping over the offsets inside one thread,
// and about 30 registers, so every SM runs its full complement of warps.
__global__ void __launch_bounds__(kQueryThreads)
kmap_probe_sym_kernel(const SlotGroup *__restrict__ groups, uint32_t cap_mask, const int4 *__restrict__ out_coords,
                      int64_t n_out, Geom g, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask,
                      int32_t *d_status) {
    pdl_enter();
    const int k = blockIdx.y;
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    if (j >= n_out) return;
    const int4 c = __ldg(out_coords + j);
    uint64_t key = 0;
    bool ok;
    if (g.shift && c.y >= g.lo[0] && c.y <= g.hi[0] && c.z >= g.lo[1] && c.z <= g.hi[1] && c.w >= g.lo[2] &&
        c.w <= g.hi[2] && pack_key(c.x, c.y, c.z, c.w, key)) {
        key += uint64_t(g.delta[k]);
        ok = true;
    } else {
        ok = query_coord(g, c, g.off[k][0], g.off[k][1], g.off[k][2], key);
    }
    int r = -1;
    if (ok) {
        uint32_t slot = probe_start(key, cap_mask);
        for (uint32_t round = 0; round < probe_window(cap_mask) / kGroupSlots; ++round) {
            const SlotGroup *gp = groups + slot / kGroupSlots;
            const ulonglong2 a = __ldg(reinterpret_cast<const ulonglong2 *>(gp->key));
            const ulonglong2 b = __ldg(reinterpret_cast<const ulonglong2 *>(gp->key + 2));
            const uint64_t k4[kGroupSlots] = {a.x, a.y, b.x, b.y};
            int found = -1;
            bool stop = false;
#pragma unroll
            for (int i = 0; i < kGroupSlots; ++i) {
                if (stop) continue;
                if (k4[i] == key) {
                    found = i;
                    stop = true;
                } else if (k4[i] == kEmptyKey) {
                    stop = true;
                }
            }
            if (stop) {
                if (found >= 0) r = int(__ldg(&gp->row[found]));
                break;
            }
            slot = (slot + kGroupSlots) & cap_mask;
        }
    }
    if (r >= n_out) {
        flag(d_status, LAT_ERR_BAD_MAP);
        r = -1;
    }
    nbr[int64_t(k) * n_out + j] = r;
    if (r >= 0) {
        const int km = g.k3 - 1 - k;
        nbr[int64_t(km) * n_out + r] = int32_t(j);
        atomicOr(mask + j, 1u << k);
        atomicOr(mask + r, 1u << km);
    }
}

// Exclusive scan of the per-block hit counts of one offset (block k scans row k of
// block_counts) -> block_offsets relative to the offset's first pair, and the
// offset's total pair count.
__global__ void __launch_bounds__(1024)
kmap_scan_kernel(const int32_t *__restrict__ block_counts, int64_t *__restrict__ block_offsets, int nblk,
                 int64_t *__restrict__ k_total) {
    pdl_enter();
    __shared__ int64_t s_warp[32];
    __shared__ int64_t s_carry;
    const int k = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int32_t *row = block_counts + int64_t(k) * nblk;
    int64_t *orow = block_offsets + int64_t(k) * nblk;
    if (t == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base < nblk; base += 1024) {
        const int e = base + t;
        const int64_t v = e < nblk ? row[e] : 0;
        int64_t incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane == 31) s_warp[w] = incl;
        __syncthreads();
        if (w == 0) {
            int64_t ws = s_warp[lane];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int64_t o = __shfl_up_sync(0xFFFFFFFFu, ws, d);
                if (lane >= d) ws += o;
            }
            s_warp[lane] = ws;
        }
        __syncthreads();
        const int64_t excl = s_carry + (w ? s_warp[w - 1] : 0) + incl - v;
        if (e < nblk) orow[e] = excl;
        __syncthreads();
        if (t == 1023) s_carry = excl + v;
        __syncthreads();
    }
    if (t == 0) k_total[k] = s_carry;
}

// Pairs of every offset at ballot-ranked positions.  The offsets a row has
// come from its mask; nbr is read only where a bit is set.
__global__ void __launch_bounds__(kQueryThreads)
kmap_emit_kernel(const int32_t *__restrict__ nbr, const uint32_t *__restrict__ mask, int64_t n_out, int k3,
                 const int64_t *__restrict__ block_offsets, const int64_t *__restrict__ k_total, int nblk,
                 int32_t *__restrict__ pair_in, int32_t *__restrict__ pair_out, int64_t capacity,
                 int64_t *__restrict__ pair_off, int32_t *d_status) {
    pdl_enter();
    __shared__ int s_warp[32][kQueryWarps];  // per (offset, warp): hits, then the exclusive prefix over warps
    __shared__ int64_t s_base[32];           // first pair of (offset, this block)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp == 0) {
        // offset starts = exclusive scan of the per-offset totals, all loads in parallel
        const int64_t tot = lane < k3 ? k_total[lane] : 0;
        const int64_t bo = lane < k3 ? block_offsets[int64_t(lane) * nblk + blockIdx.x] : 0;
        int64_t incl = tot;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane < k3) s_base[lane] = incl - tot + bo;
        if (blockIdx.x == 0) {
            if (lane < k3) pair_off[lane] = incl - tot;
            const int64_t all = __shfl_sync(0xFFFFFFFFu, incl, k3 - 1);
            if (lane == 0) pair_off[k3] = all;
        }
    }
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const uint32_t m = j < n_out ? __ldg(mask + j) : 0u;
    for (int k = 0; k < k3; ++k) {
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
        if (lane == 0) s_warp[k][warp] = __popc(hits);
    }
    __syncthreads();
    if (threadIdx.x < k3) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kQueryWarps; ++w) {
            const int c = s_warp[threadIdx.x][w];
            s_warp[threadIdx.x][w] = run;
            run += c;
        }
    }
    __syncthreads();
    bool over = false;
    for (int k = 0; k < k3; ++k) {
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
        if (!((m >> k) & 1u)) continue;
        const int64_t pos = s_base[k] + s_warp[k][warp] + __popc(hits & ((1u << lane) - 1u));
        if (pos < capacity) {
            pair_in[pos] = __ldg(nbr + int64_t(k) * n_out + j);
            pair_out[pos] = int32_t(j);
        } else {
            over = true;
        }
    }
    if (over) flag(d_status, LAT_ERR_CAPACITY);
}

// Block d: exclusive scan, in place, of digit d's per-tile counts
// hist[d * ntile + 0 .. ntile), and the digit's total into totals[d].
__global__ void __launch_bounds__(256)
sort_rowscan_kernel(int32_t *__restrict__ hist, int ntile, int32_t *__restrict__ totals) {
    pdl_enter();
    __shared__ int s_warp[8];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    int32_t *row = hist + int64_t(blockIdx.x) * ntile;
    int carry = 0;
    for (int base = 0; base < ntile; base += 256) {
        const int i = base + t;
        const int v = i < ntile ? row[i] : 0;
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane == 31) s_warp[w] = incl;
        __syncthreads();
        int before = 0, all = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int x = s_warp[q];
            before += q < w ? x : 0;
            all += x;
        }
        if (i < ntile) row[i] = carry + before + incl - v;
        carry += all;
        __syncthreads();
    }
    if (t == 0) totals[blockIdx.x] = carry;
}

// Pair lists written by the last sort pass when every row has at most one
// neighbour and the key is the one-hot mask (transposed maps from parents with
// K^3 <= 8): then the sorted order is the canonical pair order.  src == nullptr
// means no pairs here.
struct PairOut {
    const int32_t *src;  // the neighbour of each row
    int32_t *in, *out;
    int64_t capacity;
    int64_t *off;
    int k3;
    int32_t *status;
};

// One pass: scatter the rows of tile blockIdx.x by digit (key >> shift) & 255 to
// the positions `off` gives.  vals_in == nullptr means the identity (row e).
// LAST: write perm and OR masks into tile_mask; otherwise write the keys and
// rows for the next pass and count its digit per output tile into hist_next.
// All loads of the tile are issued before the first round.
template <bool LAST>
__global__ void __launch_bounds__(kSortThreads)
sort_scatter_kernel(const uint32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in, int64_t n, int shift,
                    const int32_t *__restrict__ off, const int32_t *__restrict__ totals, int ntile,
                    uint32_t *__restrict__ keys_out,
                    int32_t *__restrict__ vals_out, int32_t *__restrict__ hist_next,
                    const uint32_t *__restrict__ mask, uint32_t *__restrict__ tile_mask, PairOut po) {
    pdl_enter();
    __shared__ int s_cnt[2][kSortWarps][256];
    __shared__ int s_run[256];
    __shared__ int s_wsum[kSortWarps];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const int b = blockIdx.x;
    // first output position of digit t: exclusive scan of the digit totals
    const int tot = totals[t];  // kSortThreads == 256 digits
    const int off_b = off[int64_t(t) * ntile + b];
    uint32_t key[kSortRounds], mk[kSortRounds];
    int32_t val[kSortRounds];
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t e = int64_t(b) * kSortTile + r * kSortThreads + t;
        key[r] = 0;
        val[r] = -1;
        if (e < n) {
            key[r] = __ldg(keys_in + e);
            val[r] = vals_in ? __ldg(vals_in + e) : int32_t(e);
        }
    }
    if (LAST) {
#pragma unroll
        for (int r = 0; r < kSortRounds; ++r) mk[r] = val[r] >= 0 ? __ldg(mask + val[r]) : 0u;
    }
    for (int i = t; i < 2 * kSortWarps * 256; i += kSortThreads) (&s_cnt[0][0][0])[i] = 0;
    int incl = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int base = incl - tot;
    for (int q = 0; q < warp; ++q) base += s_wsum[q];
    s_run[t] = base + off_b;
    // one neighbour per row (po.src): rows of key 0 have none and sort first;
    // offset k's pairs are the rows of key 1 << k, in sorted order
    const int zero = po.src ? __ldg(totals) : 0;
    if (LAST && po.src && b == 0) {
        if (t > 0 && (t & (t - 1)) == 0 && __ffs(t) - 1 < po.k3) po.off[__ffs(t) - 1] = base - zero;
        if (t == 255) po.off[po.k3] = base + tot - zero;
    }
    bool over = false;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
        const int p = r & 1;
        const bool live = val[r] >= 0;
        const uint32_t d = (key[r] >> shift) & 255u;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d : 256u + lane);
        const bool leader = live && (peers & lt) == 0;
        if (leader) s_cnt[p][warp][d] = __popc(peers);
        __syncthreads();
        int64_t dst = 0;
        if (live) {
            int pre = s_run[d] + __popc(peers & lt);
            for (int w = 0; w < warp; ++w) pre += s_cnt[p][w][d];
            dst = pre;
        }
        __syncthreads();
        // digit t: advance its running position and clear this round's counts
        int add = 0;
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) {
            add += s_cnt[p][w][t];
            s_cnt[p][w][t] = 0;
        }
        s_run[t] += add;
        if (LAST) {
            if (live) vals_out[dst] = val[r];
            if (po.src && live && key[r] != 0) {
                const int64_t pos = dst - zero;
                if (pos < po.capacity) {
                    po.in[pos] = __ldg(po.src + val[r]);
                    po.out[pos] = val[r];
                } else {
                    over = true;
                }
            }
            // one atomic per (warp, output tile)
            const uint32_t tile = live ? uint32_t(dst / LAT_TILE_ROWS) : (0x80000000u | lane);
            const unsigned tp = __match_any_sync(0xFFFFFFFFu, tile);
            const uint32_t m_or = __reduce_or_sync(tp, mk[r]);
            if (live && (tp & lt) == 0) atomicOr(tile_mask + dst / LAT_TILE_ROWS, m_or);
        } else {
            if (live) {
                keys_out[dst] = key[r];
                vals_out[dst] = val[r];
            }
            const uint32_t d2 = (key[r] >> (shift + 8)) & 255u;
            // output tile < 2^31 / kSortTile <= 2^22, digit < 2^8: the tag fits in 30 bits
            const uint32_t tag = live ? ((d2 << 22) | uint32_t(dst / kSortTile)) : (0x80000000u | lane);
            const unsigned p2 = __match_any_sync(0xFFFFFFFFu, tag);
            if (live && (p2 & lt) == 0) atomicAdd(hist_next + int64_t(d2) * ntile + dst / kSortTile, int(__popc(p2)));
        }
    }
    if (over) flag(po.status, LAT_ERR_CAPACITY);
}

// Per-(offset, block) hit counts, grouping keys and the first sort pass's
// histogram from the masks (submanifold probes and maps built from parent indices).
__global__ void __launch_bounds__(kQueryThreads)
kmap_count_kernel(const uint32_t *__restrict__ mask, int64_t n_out, int k3, int32_t *__restrict__ block_counts,
                  int nblk, uint32_t *__restrict__ keys, int32_t *__restrict__ hist, int ntile) {
    pdl_enter();
    __shared__ int s_cnt[32];
    if (threadIdx.x < 32) s_cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const bool live = j < n_out;
    const uint32_t m = live ? __ldg(mask + j) : 0u;
    for (int k = 0; k < k3; ++k) {
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
        if ((threadIdx.x & 31) == 0 && hits) atomicAdd(&s_cnt[k], __popc(hits));
    }
    const uint32_t key = group_key(m, k3);
    if (live) keys[j] = key;
    sort_hist_add(key, live, j, hist, ntile);
    __syncthreads();
    if (threadIdx.x < k3) block_counts[int64_t(threadIdx.x) * nblk + blockIdx.x] = s_cnt[threadIdx.x];
}

// Kernel size == stride, no padding: fine row i lies in exactly one coarse window,
// parent[i], at offset k(i) = its position inside the window (floor modulo the
// stride per axis).  Writes the transposed map's rows directly (one neighbour per
// fine row) and scatters the strided map's entries (the down table must hold -1
// and the down mask 0 beforehand).
__global__ void __launch_bounds__(256)
parent_maps_kernel(const int4 *__restrict__ fine, const int32_t *__restrict__ parent, int64_t n_fine,
                   int64_t n_coarse, int s0, int s1, int s2, int k3, int32_t *__restrict__ up_nbr,
                   uint32_t *__restrict__ up_mask, int32_t *__restrict__ down_nbr, uint32_t *__restrict__ down_mask,
                   uint32_t *__restrict__ up_keys, int32_t *__restrict__ up_hist, int up_ntile, int32_t *d_status) {
    pdl_enter();
    const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    const bool live = i < n_fine;
    uint32_t m = 0;
    if (live) {
        const int4 c = __ldg(fine + i);
        const int q = __ldg(parent + i);
        const int o0 = c.y - floordiv(c.y, s0) * s0, o1 = c.z - floordiv(c.z, s1) * s1,
                  o2 = c.w - floordiv(c.w, s2) * s2;
        const int k = (o0 * s1 + o1) * s2 + o2;
        const bool ok = q >= 0 && q < n_coarse;
        if (!ok) flag(d_status, LAT_ERR_BAD_MAP);
        m = ok ? (1u << k) : 0u;
        if (up_nbr) {
            for (int kk = 0; kk < k3; ++kk) up_nbr[int64_t(kk) * n_fine + i] = (ok && kk == k) ? q : -1;
            up_mask[i] = m;
        }
        if (down_nbr && ok) {
            down_nbr[int64_t(k) * n_coarse + q] = int32_t(i);
            atomicOr(down_mask + q, 1u << k);
        }
    }
    // transposed map with K^3 <= 8: the grouping key is the mask, and its first
    // sort histogram is built here (every lane of the warp takes part)
    if (up_keys) {
        if (live) up_keys[i] = m;
        sort_hist_add(m, live, i, up_hist, up_ntile);
    }
}

struct KmapWs {
    int32_t *block_counts;
    int64_t *block_offsets;
    int64_t *k_total;
    uint32_t *keys;
    uint32_t *keys_tmp;
    int32_t *vals_tmp;
    int32_t *hist;    // two histograms of 256 x ntile, cleared before the keys are computed
    int32_t *totals;  // per-digit totals of each pass
    int ntile;
    size_t hist_bytes;
    size_t total;
};

static KmapWs carve_kmap_ws(void *base, int64_t n_out, int k3) {
    KmapWs w{};
    const int nblk = int((n_out + kQueryThreads - 1) / kQueryThreads);
    w.ntile = int((n_out + kSortTile - 1) / kSortTile);
    Carver cv(base);
    w.block_counts = cv.take<int32_t>(size_t(k3) * nblk);
    w.block_offsets = cv.take<int64_t>(size_t(k3) * nblk);
    w.k_total = cv.take<int64_t>(size_t(k3));
    w.keys = cv.take<uint32_t>(size_t(n_out));
    w.keys_tmp = cv.take<uint32_t>(size_t(n_out));
    w.vals_tmp = cv.take<int32_t>(size_t(n_out));
    w.hist_bytes = sizeof(int32_t) * 2 * 256 * size_t(w.ntile);
    w.hist = cv.take<int32_t>(2 * 256 * size_t(w.ntile));
    w.totals = cv.take<int32_t>(2 * 256);
    w.total = align_up(cv.used, 256);
    return w;
}

static lat_status sort_rows(lat_kmap *map, int k3, KmapWs &w, cudaStream_t s);

// Scan the per-block counts, emit the pair lists, sort the rows by grouping key
// (perm) and OR the tile masks.  The keys and the first sort histogram are in w.
// The pair chain (scan, emit) and the sort chain are independent: with a side
// stream the pair chain runs on it, concurrently with the sort on `s`.
static lat_status finish_kmap(lat_kmap *map, int k3, int nblk, KmapWs &w, int32_t *d_status, cudaStream_t s,
                              SideStream *side) {
    const int64_t n_out = map->n_out;
    cudaStream_t ps = s;
    if (side) {
        LAT_CUDA_TRY(side_fork(*side, s));
        ps = side->side;
    }
    LAT_CUDA_TRY(launch_pdl(kmap_scan_kernel, dim3(k3), dim3(1024), 0, ps, w.block_counts, w.block_offsets, nblk,
                            w.k_total));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(kmap_emit_kernel, dim3(nblk), dim3(kQueryThreads), 0, ps, map->nbr, map->mask, n_out, k3,
                            w.block_offsets, w.k_total, nblk, map->pair_in, map->pair_out, map->pair_capacity,
                            map->pair_off, d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    const lat_status st = sort_rows(map, k3, w, s);
    if (side) LAT_CUDA_TRY(side_join(*side, s));
    return st;
}

// Stable row sort by grouping key -> perm, tile masks ORed by the last pass
// (map->tile_mask must hold zeros beforehand).
static lat_status sort_rows(lat_kmap *map, int k3, KmapWs &w, cudaStream_t s) {
    const int64_t n_out = map->n_out;
    const int64_t hsize = 256 * int64_t(w.ntile);
    int32_t *h1 = w.hist, *h2 = w.hist + hsize;
    int32_t *t1 = w.totals, *t2 = w.totals + 256;
    LAT_CUDA_TRY(launch_pdl(sort_rowscan_kernel, dim3(256), dim3(256), 0, s, h1, w.ntile, t1));
    LAT_CUDA_TRY(cudaGetLastError());
    if (group_key_bits(k3) <= 8) {
        LAT_CUDA_TRY(launch_pdl(sort_scatter_kernel<true>, dim3(w.ntile), dim3(kSortThreads), 0, s, w.keys, nullptr,
                                n_out, 0, h1, t1, w.ntile, nullptr, map->perm, nullptr, map->mask, map->tile_mask,
                                PairOut{}));
        LAT_CUDA_TRY(cudaGetLastError());
        return LAT_OK;
    }
    LAT_CUDA_TRY(launch_pdl(sort_scatter_kernel<false>, dim3(w.ntile), dim3(kSortThreads), 0, s, w.keys, nullptr,
                            n_out, 0, h1, t1, w.ntile, w.keys_tmp, w.vals_tmp, h2, nullptr, nullptr, PairOut{}));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(sort_rowscan_kernel, dim3(256), dim3(256), 0, s, h2, w.ntile, t2));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(sort_scatter_kernel<true>, dim3(w.ntile), dim3(kSortThreads), 0, s, w.keys_tmp, w.vals_tmp,
                            n_out, 8, h2, t2, w.ntile, nullptr, map->perm, nullptr, map->mask, map->tile_mask,
                            PairOut{}));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}

static bool map_buffers_ok(const lat_kmap *map) {
    if (!map || map->n_out < 0 || map->n_out >= (int64_t(1) << 31) || map->n_in < 0 ||
        map->n_in >= (int64_t(1) << 31) || map->pair_capacity < 0 || !map->pair_off)
        return false;
    if (map->n_out > 0 && (!map->nbr || !map->mask || !map->perm || !map->tile_mask)) return false;
    if (map->pair_capacity > 0 && (!map->pair_in || !map->pair_out)) return false;
    return true;
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
    if (!map || !geom_ok(geom, k3) || map->k3 != k3 || !map_buffers_ok(map)) return LAT_ERR_ARG;
    const int64_t n_out = map->n_out, n_in = map->n_in;
    if (!table || table_bytes % kSlotBytes || !pow2(table_bytes / kSlotBytes) || table_bytes / kSlotBytes < 64 ||
        table_bytes / kSlotBytes > (uint64_t(1) << 31))
        return LAT_ERR_ARG;
    if (n_out > 0 && !out_coords) return LAT_ERR_ARG;
    if (geom->mode == LAT_SUBM && n_in != n_out) return LAT_ERR_ARG;  // the support is preserved
    if (reinterpret_cast<uintptr_t>(out_coords) % 16 || reinterpret_cast<uintptr_t>(table) % 64) return LAT_ERR_ARG;
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
    // unit stride: probed coordinate = own + sign * (off - pad), sign -1 for the transposed relation
    g.shift = g.st[0] == 1 && g.st[1] == 1 && g.st[2] == 1;
    const int sign = g.mode == LAT_TRANSPOSED ? -1 : 1;
    int dmin[3] = {0, 0, 0}, dmax[3] = {0, 0, 0};
    for (int a = 0; a < 3; ++a) {
        const int d0 = sign * (0 - g.pd[a]), d1 = sign * (g.ks[a] - 1 - g.pd[a]);
        dmin[a] = d0 < d1 ? d0 : d1;
        dmax[a] = d0 < d1 ? d1 : d0;
        g.lo[a] = -32768 - dmin[a];
        g.hi[a] = 32767 - dmax[a];
    }
    for (int ix = 0, k = 0; ix < g.ks[0]; ++ix)
        for (int iy = 0; iy < g.ks[1]; ++iy)
            for (int iz = 0; iz < g.ks[2]; ++iz, ++k) {
                g.off[k][0] = static_cast<signed char>(ix);
                g.off[k][1] = static_cast<signed char>(iy);
                g.off[k][2] = static_cast<signed char>(iz);
                const long long dx = sign * (ix - g.pd[0]), dy = sign * (iy - g.pd[1]), dz = sign * (iz - g.pd[2]);
                g.delta[k] = dx * (1ll << 32) + dy * (1ll << 16) + dz;
            }
    const int nblk = int((n_out + kQueryThreads - 1) / kQueryThreads);
    const int64_t ntiles = (n_out + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS;
    const uint32_t cap_mask = uint32_t(table_bytes / kSlotBytes - 1);
    const SlotGroup *slots = static_cast<const SlotGroup *>(table);
    const int4 *oc = reinterpret_cast<const int4 *>(out_coords);
    if (geom->mode == LAT_SUBM) {
        // the upper half of the table is filled by mirrored hits only
        const int centre = k3 / 2;
        LAT_CUDA_TRY(launch_pdl(kmap_subm_init_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, n_out, k3, map->nbr,
                                map->mask, w.hist, int64_t(w.hist_bytes / 4), map->tile_mask, ntiles));
        LAT_CUDA_TRY(cudaGetLastError());
        if (centre > 0) {
            LAT_CUDA_TRY(launch_pdl(kmap_probe_sym_kernel, dim3(unsigned(nblk), unsigned(centre)), dim3(kQueryThreads),
                                    0, s, slots, cap_mask, oc, n_out, g, map->nbr, map->mask, d_status));
            LAT_CUDA_TRY(cudaGetLastError());
        }
        LAT_CUDA_TRY(launch_pdl(kmap_count_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, map->mask, n_out, k3,
                                w.block_counts, nblk, w.keys, w.hist, w.ntile));
    } else {
        FillList f;
        f.add(w.hist, int64_t(w.hist_bytes / 4), 0u);
        f.add(map->tile_mask, ntiles, 0u);
        LAT_CUDA_TRY(fill_list(f, s));
        LAT_CUDA_TRY(launch_pdl(kmap_probe_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, slots, cap_mask, oc, n_out,
                                n_in, g, map->nbr, map->mask, w.keys, w.hist, w.ntile, w.block_counts, nblk, d_status));
    }
    LAT_CUDA_TRY(cudaGetLastError());
    SideStream *side = nullptr;
    LAT_CUDA_TRY(side_stream(side));
    return finish_kmap(map, k3, nblk, w, d_status, s, side);
}

extern "C" size_t lat_kmap_from_parent_ws_bytes(int64_t n_fine, int64_t n_coarse, int32_t k3) {
    if (n_fine < 0 || n_coarse < 0 || n_fine >= (int64_t(1) << 31) || k3 < 1 || k3 > 32) return 0;
    // the strided map's workspace, then the transposed map's (its keys are built
    // before the strided map is finished)
    return lat::carve_kmap_ws(nullptr, n_coarse, k3).total + lat::carve_kmap_ws(nullptr, n_fine, k3).total;
}

extern "C" lat_status lat_kmap_from_parent(const int32_t *fine_coords, const int32_t *parent, const lat_geom *geom,
                                           lat_kmap *down, lat_kmap *up, void *ws, size_t ws_bytes,
                                           int32_t *d_status, lat_stream stream) {
    using namespace lat;
    int k3 = 0;
    if (!geom_ok(geom, k3) || geom->mode != LAT_STRIDED) return LAT_ERR_ARG;
    for (int a = 0; a < 3; ++a)
        if (geom->ksize[a] != geom->stride[a] || geom->pad[a] != 0) return LAT_ERR_UNSUPPORTED;
    if (!down && !up) return LAT_ERR_ARG;
    if ((down && (!map_buffers_ok(down) || down->k3 != k3)) || (up && (!map_buffers_ok(up) || up->k3 != k3)))
        return LAT_ERR_ARG;
    const int64_t n_fine = up ? up->n_out : down->n_in;
    const int64_t n_coarse = up ? up->n_in : down->n_out;
    if (down && up && (down->n_in != n_fine || down->n_out != n_coarse)) return LAT_ERR_ARG;
    if (n_fine > 0 && (!fine_coords || !parent)) return LAT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(fine_coords) % 16) return LAT_ERR_ARG;
    const size_t need = lat_kmap_from_parent_ws_bytes(n_fine, n_coarse, k3);
    if (ws_bytes < need || (need && !ws)) return LAT_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (down) down->mode = LAT_STRIDED;
    if (up) up->mode = LAT_TRANSPOSED;
    KmapWs w_down = carve_kmap_ws(ws, n_coarse, k3);
    KmapWs w_up = carve_kmap_ws(static_cast<char *>(ws) + w_down.total, n_fine, k3);
    // transposed map with K^3 <= 8: every fine row has one neighbour (its parent)
    // and its key is the one-hot mask, so the row sort alone yields the pairs
    const bool up_direct = up && n_fine > 0 && group_key_bits(k3) <= 8;
    // every initialisation both maps need, in one launch: the strided map's
    // table (-1) and masks (0, both filled by the parent scatter), and each
    // map's sort histograms and tile masks
    FillList f;
    if (down && n_coarse > 0) {
        f.add(down->nbr, int64_t(k3) * n_coarse, ~0u);
        f.add(down->mask, n_coarse, 0u);
        f.add(w_down.hist, int64_t(w_down.hist_bytes / 4), 0u);
        f.add(down->tile_mask, (n_coarse + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS, 0u);
    }
    if (up && n_fine > 0) {
        f.add(w_up.hist, int64_t(w_up.hist_bytes / 4), 0u);
        f.add(up->tile_mask, (n_fine + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS, 0u);
    }
    LAT_CUDA_TRY(fill_list(f, s));
    if (n_fine > 0) {
        LAT_CUDA_TRY(launch_pdl(parent_maps_kernel, dim3(unsigned((n_fine + 255) / 256)), dim3(256), 0, s,
                                reinterpret_cast<const int4 *>(fine_coords), parent, n_fine, n_coarse, geom->stride[0],
                                geom->stride[1], geom->stride[2], k3, up ? up->nbr : nullptr, up ? up->mask : nullptr,
                                down ? down->nbr : nullptr, down ? down->mask : nullptr,
                                up_direct ? w_up.keys : nullptr, w_up.hist, w_up.ntile, d_status));
        LAT_CUDA_TRY(cudaGetLastError());
    }
    // the two maps are independent once the parent scatter is done: the
    // transposed one is finished on a side stream, concurrently with the other
    SideStream *side = nullptr;
    if (down && up) {
        LAT_CUDA_TRY(side_stream(side));
        LAT_CUDA_TRY(side_fork(*side, s));
    }
    const cudaStream_t main_s = s;
    for (lat_kmap *map : {down, up}) {
        if (!map) continue;
        const cudaStream_t s = (side && map == up) ? side->side : main_s;
        if (map->n_out == 0) {
            LAT_CUDA_TRY(cudaMemsetAsync(map->pair_off, 0, sizeof(int64_t) * (k3 + 1), s));
            continue;
        }
        KmapWs &w = map == down ? w_down : w_up;
        if (map == up && up_direct) {
            LAT_CUDA_TRY(launch_pdl(sort_rowscan_kernel, dim3(256), dim3(256), 0, s, w.hist, w.ntile, w.totals));
            LAT_CUDA_TRY(cudaGetLastError());
            const PairOut po{parent, map->pair_in, map->pair_out, map->pair_capacity, map->pair_off, k3, d_status};
            LAT_CUDA_TRY(launch_pdl(sort_scatter_kernel<true>, dim3(w.ntile), dim3(kSortThreads), 0, s, w.keys,
                                    nullptr, map->n_out, 0, w.hist, w.totals, w.ntile, nullptr, map->perm, nullptr,
                                    map->mask, map->tile_mask, po));
            LAT_CUDA_TRY(cudaGetLastError());
            continue;
        }
        const int nblk = int((map->n_out + kQueryThreads - 1) / kQueryThreads);
        LAT_CUDA_TRY(launch_pdl(kmap_count_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, map->mask, map->n_out, k3,
                                w.block_counts, nblk, w.keys, w.hist, w.ntile));
        LAT_CUDA_TRY(cudaGetLastError());
        const lat_status st = finish_kmap(map, k3, nblk, w, d_status, s, nullptr);
        if (st != LAT_OK) return st;
    }
    if (side) LAT_CUDA_TRY(side_join(*side, main_s));
    return LAT_OK;
}
