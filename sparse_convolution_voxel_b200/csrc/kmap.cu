// Kernel-map construction / coordinate query (lat_kmap_ws_bytes, lat_kmap_query,
// lat_kmap_from_parent).
//
// Torch Lattice docs, "Migrating from TorchSparse": kernel-map construction
// and coordinate query are CUDA kernels of the library ("What remains
// familiar", "Sparse tensor expectations"), and the support semantics come
// from the "Convolution mapping" table.  Pipeline of one map (all on
// `stream`; four launches for a submanifold map with K^3 > 8):
//   0. fill:   zeroes the global counters, the sweeps' look-back state and
//              the tile masks.
//   1. front end: nbr (offset-major), the neighbour mask and the grouping key
//              of every output row, plus global totals: hits per offset and
//              the histograms of both bytes of the key.
//                submanifold maps:  subm_probe_kernel (one warp per kernel
//                                   column (ix, iy); one probe of a z-brick
//                                   answers the column's Kz offsets)
//                strided/transposed: kmap_probe_kernel (a row per thread)
//                maps from parents: parent_maps_kernel (+ kmap_count_kernel)
//   2. sweep 1: the pair lists (grouped by offset, output rows ascending) and
//              the first stable radix pass of the rows by the key's low byte.
//   3. sweep 2: the second pass (high byte) -> perm, and the tile masks.
//              With K^3 <= 8 the key is the mask itself (one byte) and
//              sweep 1 writes perm and the tile masks directly.
// The sweeps cut the rows into tiles of kSwTile positions; a tile learns
// where its rows go from its predecessors' counts by decoupled look-back
// (Merrill and Garland, "Single-pass Parallel Prefix Scan with Decoupled
// Look-back", 2016; Adinets and Merrill's one-sweep radix sort uses it once
// per digit): it publishes its own counts, then walks back over the earlier
// tiles until it meets one that has published an inclusive prefix.  Tiles
// are numbered in the order blocks start, so every tile it waits for is
// already running; every wait is bounded.  Ranks inside a tile keep row
// order, so the sort is stable and every output is deterministic.
#include "common.cuh"

namespace lat {

constexpr int kQueryThreads = 256;

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
__host__ __device__ inline int group_key_bits(int k3) { return k3 <= 8 ? k3 : kGroupKeyBits; }

// ----------------------------------------------------------------------------- global totals
// counters[0..255]: histogram of the key's low byte, [256..511]: of its high
// byte, [512..543]: hits per offset, [544], [545]: tile counters of the two
// sweeps.  Zero before the front end runs.
constexpr int kCntHist = 0, kCntOff = 512, kCntTile = 544, kCntWords = 576;

// Shared-memory tallies of one block (s_h: both key-byte histograms, s_o: hits
// per offset), added to the global counters once at the end of the block.
struct Tally {
    int *s_h;  // [512]
    int *s_o;  // [32]
};

// Counts one row per lane into the block's tallies; every lane of the warp calls it.
__device__ __forceinline__ void tally_row(const Tally &ty, uint32_t key, uint32_t m, bool live, bool two) {
    const int lane = threadIdx.x & 31;
    const uint32_t d0 = key & 255u;
    unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d0 : 256u + lane);
    if (live && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&ty.s_h[d0], int(__popc(peers)));
    if (two) {
        const uint32_t d1 = (key >> 8) & 255u;
        peers = __match_any_sync(0xFFFFFFFFu, live ? d1 : 256u + lane);
        if (live && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&ty.s_h[256 + d1], int(__popc(peers)));
    }
    const uint32_t mm = live ? m : 0u;
    for (uint32_t any = __reduce_or_sync(0xFFFFFFFFu, mm); any; any &= any - 1) {
        const int k = __ffs(any) - 1;
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, (mm >> k) & 1u);
        if (lane == 0) atomicAdd(&ty.s_o[k], int(__popc(hits)));
    }
}

__device__ __forceinline__ void tally_clear(const Tally &ty) {
    for (int i = threadIdx.x; i < 512 + 32; i += blockDim.x) (i < 512 ? ty.s_h[i] : ty.s_o[i - 512]) = 0;
}

// Adds the block's tallies to the global counters (after a __syncthreads()).
__device__ __forceinline__ void tally_flush(const Tally &ty, int k3, bool two, int32_t *counters) {
    for (int i = threadIdx.x; i < 512 + 32; i += blockDim.x) {
        if (i < 512) {
            const int v = ty.s_h[i];
            if (v && (i < 256 || two)) atomicAdd(counters + kCntHist + i, v);
        } else if (i - 512 < k3) {
            const int v = ty.s_o[i - 512];
            if (v) atomicAdd(counters + kCntOff + (i - 512), v);
        }
    }
}

// ----------------------------------------------------------------------------- table lookups
// The 4 keys of the slot group holding slot s (two 16-byte loads of one sector).
__device__ __forceinline__ void group_keys(const SlotGroup *groups, uint32_t s, uint64_t (&k4)[kGroupSlots]) {
    const SlotGroup *gp = groups + s / kGroupSlots;
    const ulonglong2 a = __ldg(reinterpret_cast<const ulonglong2 *>(gp->key));
    const ulonglong2 b = __ldg(reinterpret_cast<const ulonglong2 *>(gp->key + 2));
    k4[0] = a.x;
    k4[1] = a.y;
    k4[2] = b.x;
    k4[3] = b.y;
}

// Slot of `key` (linear probing from its group start), -1 if absent.
__device__ __forceinline__ int probe_one(const SlotGroup *groups, uint32_t cap_mask, uint64_t key) {
    uint32_t slot = probe_start(key, cap_mask);
    for (uint32_t round = 0; round < probe_window(cap_mask) / kGroupSlots; ++round) {
        uint64_t k4[kGroupSlots];
        group_keys(groups, slot, k4);
#pragma unroll
        for (int i = 0; i < kGroupSlots; ++i) {
            if (k4[i] == key) return int(slot) + i;
            if (k4[i] == kEmptyKey) return -1;
        }
        slot = (slot + kGroupSlots) & cap_mask;
    }
    return -1;
}

// Searches one kernel column (b, X, Y) for its KZ targets z_t = zlo + t
// (t = 0..KZ-1, bit t of `want` set for the ones to look up), given as the
// column's upper key word col_hi = b<<16 | X field, the Y field and the z
// field zf0 of target 0.  A slot holds target t iff its upper 48 bits equal
// the column's and its z field is zf0 + t.  Every key lives in the probe
// sequence of its z-brick (probe_start ignores the low two bits of the z
// field), so KZ <= 5 consecutive targets need at most two sequences, A for
// the first wanted target's brick and B for the last's; both are read at once
// and each is walked until its targets are found or it shows an empty slot
// (no key of that brick lies beyond an empty slot of its sequence).  Bounded
// by the probe window.  slot_of[t] = the slot of target t, or -1.
template <int KZ>
__device__ __forceinline__ void probe_column(const SlotGroup *groups, uint32_t cap_mask, uint32_t col_hi,
                                             uint32_t col_y, int zf0, uint32_t want, int (&slot_of)[KZ]) {
    static_assert(KZ >= 1 && KZ <= 5, "two z-bricks at most");
#pragma unroll
    for (int t = 0; t < KZ; ++t) slot_of[t] = -1;
    if (!want) return;
    const int t_lo = __ffs(want) - 1, t_hi = 31 - __clz(want);
    const uint32_t b_lo = uint32_t(zf0 + t_lo) >> 2, b_hi = uint32_t(zf0 + t_hi) >> 2;
    const uint64_t colkey = (uint64_t(col_hi) << 32) | (uint64_t(col_y) << 16);
    uint32_t want_a = 0;
#pragma unroll
    for (int t = 0; t < KZ; ++t)
        if (((want >> t) & 1u) && (uint32_t(zf0 + t) >> 2) == b_lo) want_a |= 1u << t;
    const uint32_t want_b = want & ~want_a;
    uint32_t sa = probe_start(colkey | (uint64_t(b_lo) << 2), cap_mask);
    uint32_t sb = probe_start(colkey | (uint64_t(b_hi) << 2), cap_mask);
    bool act_a = want_a != 0, act_b = want_b != 0;
    uint32_t found = 0;
    auto scan = [&](const uint64_t (&k4)[kGroupSlots], uint32_t s) -> bool {
        bool empty = false;
#pragma unroll
        for (int i = 0; i < kGroupSlots; ++i) {
            const uint64_t k = k4[i];
            if (k == kEmptyKey) {
                empty = true;
                continue;
            }
            if (uint32_t(k >> 32) != col_hi || uint32_t(k >> 16 & 0xFFFFu) != col_y) continue;
            const int d = int(k & 0xFFFFu) - zf0;
#pragma unroll
            for (int t = 0; t < KZ; ++t)
                if (d == t) slot_of[t] = int(s) + i;
            if (d >= 0 && d < KZ) found |= 1u << d;
        }
        return empty;
    };
    for (uint32_t round = 0; (act_a || act_b) && round < probe_window(cap_mask) / kGroupSlots; ++round) {
        uint64_t ka[kGroupSlots], kb[kGroupSlots];
        if (act_a) group_keys(groups, sa, ka);
        if (act_b) group_keys(groups, sb, kb);
        if (act_a) {
            const bool e = scan(ka, sa);
            act_a = !e && (want_a & ~found);
            sa = (sa + kGroupSlots) & cap_mask;
        }
        if (act_b) {
            const bool e = scan(kb, sb);
            act_b = !e && (want_b & ~found);
            sb = (sb + kGroupSlots) & cap_mask;
        }
    }
#pragma unroll
    for (int t = 0; t < KZ; ++t)
        if (!((want >> t) & 1u)) slot_of[t] = -1;
}

// ----------------------------------------------------------------------------- submanifold front end
struct SubmGeom {
    int kx, ky, kz;
    int px, py, pz;  // (K - 1) / 2
    int k3;
};

constexpr int kProbeRows = 128;  // output rows per block (four per lane)

// Submanifold map, one launch: block = one warp per kernel column (ix, iy)
// (warp w = ix * Ky + iy) over kProbeRows rows; the column's offsets are
// k = w * Kz + iz.  The block's coordinates are staged in shared memory once.
// A lane takes its rows one at a time: it searches the table for the
// neighbours at (x + ix - px, y + iy - py, z + iz - pz), iz = 0..Kz-1, in
// one pass over at most two z-brick sequences (KZ = 1 or 3; KZ = 0 probes
// each offset on its own, for any Kz), writes those Kz entries of nbr
// (coalesced: the warp's 32 rows are consecutive) and ballots its hits into
// shared memory.  The centre offset is the row itself and is not probed.
// Then each row's mask is gathered from the ballots, and the row's grouping
// key, the block's hits per offset and its key-byte histograms are computed
// and added to the global counters.
template <int KZ>
__global__ void __launch_bounds__(1024)
subm_probe_kernel(const SlotGroup *__restrict__ groups, uint32_t cap_mask, const int4 *__restrict__ coords, int64_t n,
                  SubmGeom g, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask, uint32_t *__restrict__ keys,
                  int32_t *__restrict__ counters, int32_t *d_status) {
    pdl_enter();
    __shared__ int4 s_c[kProbeRows];
    __shared__ uint32_t s_bits[32][kProbeRows / 32];
    __shared__ int s_h[512], s_o[32];
    const Tally ty{s_h, s_o};
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nwarp = blockDim.x >> 5;
    const int64_t row0 = int64_t(blockIdx.x) * kProbeRows;
    for (int i = tid; i < kProbeRows; i += blockDim.x)
        s_c[i] = row0 + i < n ? __ldg(coords + row0 + i) : make_int4(-1, 0, 0, 0);
    for (int i = tid; i < 32 * (kProbeRows / 32); i += blockDim.x) (&s_bits[0][0])[i] = 0u;
    tally_clear(ty);
    __syncthreads();
    const int kz = KZ ? KZ : g.kz;
    const int dx = w / g.ky - g.px, dy = w % g.ky - g.py;
    const bool own = dx == 0 && dy == 0;
    int32_t bad = 0;
    for (int r = 0; r < kProbeRows / 32; ++r) {
        const int64_t j = row0 + 32 * r + lane;
        const bool live = j < n;
        const int4 c = s_c[32 * r + lane];
        const int X = c.y + dx, Y = c.z + dy;
        const bool colok = live && c.x >= 0 && c.x <= 65534 && X >= -32768 && X <= 32767 && Y >= -32768 &&
                           Y <= 32767 && c.w >= -32768 && c.w <= 32767;
        const int zf0 = c.w + 32768 - g.pz;  // z field of target iz = 0
        const uint32_t col_hi = (uint32_t(c.x) << 16) | uint32_t(X + 32768);
        const uint32_t col_y = uint32_t(Y + 32768);
        uint32_t want = 0;
        for (int t = 0; t < kz; ++t)
            if (colok && zf0 + t >= 0 && zf0 + t <= 65535 && !(own && t == g.pz)) want |= 1u << t;
        if constexpr (KZ > 0) {
            int slot_of[KZ];
            probe_column<KZ>(groups, cap_mask, col_hi, col_y, zf0, want, slot_of);
            int rr[KZ];
#pragma unroll
            for (int t = 0; t < KZ; ++t)
                rr[t] = slot_of[t] >= 0 ? int(__ldg(&groups[slot_of[t] / kGroupSlots].row[slot_of[t] % kGroupSlots]))
                                        : -1;
#pragma unroll
            for (int t = 0; t < KZ; ++t) {
                int v = rr[t];
                if (own && t == g.pz) v = live ? int(j) : -1;
                if (v >= n) {
                    bad |= LAT_ERR_BAD_MAP;
                    v = -1;
                }
                const int k = w * KZ + t;
                if (live) nbr[int64_t(k) * n + j] = v;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, v >= 0);
                if (lane == 0) s_bits[k][r] = hits;
            }
        } else {
            for (int t = 0; t < kz; ++t) {
                int v = -1;
                if (own && t == g.pz) {
                    v = live ? int(j) : -1;
                } else if ((want >> t) & 1u) {
                    const uint64_t key = (uint64_t(col_hi) << 32) | (uint64_t(col_y) << 16) | uint64_t(zf0 + t);
                    const int s = probe_one(groups, cap_mask, key);
                    v = s >= 0 ? int(__ldg(&groups[s / kGroupSlots].row[s % kGroupSlots])) : -1;
                }
                if (v >= n) {
                    bad |= LAT_ERR_BAD_MAP;
                    v = -1;
                }
                const int k = w * kz + t;
                if (live) nbr[int64_t(k) * n + j] = v;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, v >= 0);
                if (lane == 0) s_bits[k][r] = hits;
            }
        }
    }
    if (bad) flag(d_status, bad);
    __syncthreads();
    const bool two = group_key_bits(g.k3) > 8;
    for (int r = w; r < kProbeRows / 32; r += nwarp) {
        const int64_t j = row0 + 32 * r + lane;
        const bool live = j < n;
        uint32_t m = 0;
        for (int k = 0; k < g.k3; ++k) m |= ((s_bits[k][r] >> lane) & 1u) << k;
        const uint32_t key = group_key(m, g.k3);
        if (live) {
            mask[j] = m;
            keys[j] = key;
        }
        tally_row(ty, key, m, live, two);
    }
    __syncthreads();
    tally_flush(ty, g.k3, two, counters);
}

// ----------------------------------------------------------------------------- strided / transposed front end
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
// one round.  Rounds are bounded by the probe window (kMaxProbeSlots).  Strided
// and transposed maps (and TargetConv3d's stride-1 strided maps): every
// offset is probed, and the mask, grouping key and global totals are
// produced here.
__global__ void __launch_bounds__(kQueryThreads)
kmap_probe_kernel(const SlotGroup *__restrict__ groups, uint32_t cap_mask, const int4 *__restrict__ out_coords,
                  int64_t n_out, int64_t n_in, Geom g, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask,
                  uint32_t *__restrict__ keys, int32_t *__restrict__ counters, int32_t *d_status) {
    pdl_enter();
    __shared__ int s_h[512], s_o[32];
    const Tally ty{s_h, s_o};
    tally_clear(ty);
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
            if (r >= n_in) {
                bad |= LAT_ERR_BAD_MAP;
                r = -1;
            }
            if (live) nbr[int64_t(k) * n_out + j] = r;
            if (r >= 0) m |= 1u << k;
        }
    }
    if (bad) flag(d_status, bad);
    const uint32_t key = group_key(m, g.k3);
    if (live) {
        mask[j] = m;
        keys[j] = key;
    }
    const bool two = group_key_bits(g.k3) > 8;
    tally_row(ty, key, m, live, two);
    __syncthreads();
    tally_flush(ty, g.k3, two, counters);
}

// Grouping keys and global totals from final masks (the strided map of a
// ksize == stride convolution, whose masks the parent scatter builds).
__global__ void __launch_bounds__(kQueryThreads)
kmap_count_kernel(const uint32_t *__restrict__ mask, int64_t n_out, int k3, uint32_t *__restrict__ keys,
                  int32_t *__restrict__ counters) {
    pdl_enter();
    __shared__ int s_h[512], s_o[32];
    const Tally ty{s_h, s_o};
    tally_clear(ty);
    __syncthreads();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const bool live = j < n_out;
    const uint32_t m = live ? __ldg(mask + j) : 0u;
    const uint32_t key = group_key(m, k3);
    if (live) keys[j] = key;
    const bool two = group_key_bits(k3) > 8;
    tally_row(ty, key, m, live, two);
    __syncthreads();
    tally_flush(ty, k3, two, counters);
}

// Kernel size == stride, no padding: fine row i lies in exactly one coarse window,
// parent[i], at offset k(i) = its position inside the window (floor modulo the
// stride per axis).  Writes the transposed map's rows directly (one neighbour
// per fine row), with their grouping keys and totals, and scatters the strided
// map's entries (its table must hold -1 and its masks 0 beforehand).
__global__ void __launch_bounds__(256)
parent_maps_kernel(const int4 *__restrict__ fine, const int32_t *__restrict__ parent, int64_t n_fine,
                   int64_t n_coarse, int s0, int s1, int s2, int k3, int32_t *__restrict__ up_nbr,
                   uint32_t *__restrict__ up_mask, uint32_t *__restrict__ up_keys, int32_t *__restrict__ up_counters,
                   int32_t *__restrict__ down_nbr, uint32_t *__restrict__ down_mask, int32_t *d_status) {
    pdl_enter();
    __shared__ int s_h[512], s_o[32];
    const Tally ty{s_h, s_o};
    if (up_nbr) tally_clear(ty);
    __syncthreads();
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
    if (up_nbr) {  // block-uniform: every lane of the warp takes part
        const uint32_t key = group_key(m, k3);
        if (live) up_keys[i] = key;
        const bool two = group_key_bits(k3) > 8;
        tally_row(ty, key, m, live, two);
        __syncthreads();
        tally_flush(ty, k3, two, up_counters);
    }
}

// ----------------------------------------------------------------------------- sweeps
constexpr int kSwThreads = 512;
constexpr int kSwWarps = kSwThreads / 32;
constexpr int kSwRounds = 4;
constexpr int kSwTile = kSwThreads * kSwRounds;  // rows per tile
constexpr int kSwChains = 256 + 32;              // look-back chains per tile: 256 digits, then 32 offsets
constexpr unsigned long long kFlagAgg = 1ull << 32, kFlagPrefix = 2ull << 32;
constexpr uint64_t kLookbackNs = 1000000000ull;  // a look-back wait gives up after 1 s

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

struct Sweep {
    const uint32_t *keys_in;   // key of each input position
    const int32_t *vals_in;    // output row of each input position; nullptr = the position itself
    const uint32_t *masks_in;  // neighbour mask of each input position
    int64_t n;
    int shift;                 // this pass's digit: (key >> shift) & 255
    int32_t *counters;         // global totals (kCnt*); tile counter of this sweep at kCntTile + which
    int which;                 // 0 = first sweep, 1 = second
    unsigned long long *status;  // [ntile][kSwChains] look-back words, zero at launch
    // pair emission (first sweep)
    const int32_t *nbr;
    int centre;  // offset whose neighbour of row j is j itself (submanifold), else -1
    int k3;
    int32_t *pair_in, *pair_out;
    int64_t capacity;
    int64_t *pair_off;
    // outputs: to the second sweep, or perm and the tile masks
    uint32_t *keys_out;
    int32_t *vals_out;
    uint32_t *masks_out;
    int32_t *perm;
    uint32_t *tile_mask;  // zero at launch
    int32_t *d_status;
};

// One tile of one radix pass.  EMIT: also write the pair lists (first sweep,
// rows in input order).  LAST: write perm and OR each row's mask into its
// LAT_TILE_ROWS output tile; otherwise hand (key, row, mask) to the next
// sweep at the sorted position.  Positions: the digit's start (exclusive scan
// of the global digit histogram) + the digit's count in earlier tiles
// (look-back) + the row's rank among this tile's rows of that digit (warp
// match, per-warp counts; rounds in row order).  Pair positions likewise per
// offset.
template <bool EMIT, bool LAST>
__global__ void __launch_bounds__(kSwThreads) sweep_kernel(Sweep a) {
    pdl_enter();
    __shared__ int s_tile;
    __shared__ int s_cnt[2][kSwWarps][256];  // per round (double buffered): per-warp digit counts
    __shared__ int s_run[256];               // next position of each digit
    __shared__ int s_hist[256];              // this tile's rows per digit
    __shared__ int s_ocnt[32];               // this tile's pairs per offset
    __shared__ int s_pw[2][kSwWarps][32];    // per round: per-warp pairs per offset, then their prefix
    __shared__ long long s_orun[2][32];      // per round: next pair position of each offset
    __shared__ int s_wsum[8];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const unsigned lt = (1u << lane) - 1u;
    if (t == 0) s_tile = atomicAdd(a.counters + kCntTile + a.which, 1);
    for (int i = t; i < 2 * kSwWarps * 256; i += kSwThreads) (&s_cnt[0][0][0])[i] = 0;
    if (t < 256) s_hist[t] = 0;
    if (t < 32) s_ocnt[t] = 0;
    __syncthreads();
    const int tile = s_tile;
    if (int64_t(tile) * kSwTile >= a.n) {  // the tile counter was not cleared: no tile waits for this one
        if (t == 0) flag(a.d_status, LAT_ERR_BAD_MAP);
        return;
    }
    uint32_t key[kSwRounds], mk[kSwRounds];
    int32_t val[kSwRounds];
#pragma unroll
    for (int r = 0; r < kSwRounds; ++r) {
        const int64_t e = int64_t(tile) * kSwTile + r * kSwThreads + t;
        key[r] = 0;
        mk[r] = 0;
        val[r] = -1;
        if (e < a.n) {
            key[r] = __ldg(a.keys_in + e);
            val[r] = a.vals_in ? __ldg(a.vals_in + e) : int32_t(e);
            if (EMIT || LAST) mk[r] = __ldg(a.masks_in + e);
        }
    }
    // this tile's counts
#pragma unroll
    for (int r = 0; r < kSwRounds; ++r) {
        const bool live = val[r] >= 0;
        const uint32_t d = (key[r] >> a.shift) & 255u;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d : 256u + lane);
        if (live && (peers & lt) == 0) atomicAdd(&s_hist[d], int(__popc(peers)));
        if (EMIT) {
            const uint32_t m = live ? mk[r] : 0u;
            for (uint32_t any = __reduce_or_sync(0xFFFFFFFFu, m); any; any &= any - 1) {
                const int k = __ffs(any) - 1;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
                if (lane == 0) atomicAdd(&s_ocnt[k], int(__popc(hits)));
            }
        }
    }
    __syncthreads();
    // publish this tile's counts, look back for the earlier tiles', publish the prefix
    const int nchain = EMIT ? 256 + a.k3 : 256;
    unsigned long long *st = a.status + int64_t(tile) * kSwChains;
    int own = 0, excl = 0;
    if (t < nchain) {
        own = t < 256 ? s_hist[t] : s_ocnt[t - 256];
        st_relaxed(st + t, (tile == 0 ? kFlagPrefix : kFlagAgg) | uint32_t(own));
        if (tile > 0) {
            bool timed_out = false;
            uint64_t t0 = 0;
            int64_t pb = tile - 1;
            for (uint32_t spin = 0;;) {
                const unsigned long long v = ld_relaxed(a.status + pb * kSwChains + t);
                if ((v >> 32) == 0) {  // that tile has not published yet: it is running, wait
                    if (++spin == 64) t0 = ptx_globaltimer();
                    if (spin > 64 && (spin & 15) == 0 && ptx_globaltimer() - t0 > kLookbackNs) {
                        timed_out = true;
                        break;
                    }
                    __nanosleep(64);
                    continue;
                }
                excl += int(uint32_t(v));
                if ((v >> 32) == 2 || pb == 0) break;
                --pb;
            }
            if (timed_out) flag(a.d_status, LAT_ERR_TIMEOUT);
            st_relaxed(st + t, kFlagPrefix | uint32_t(excl + own));
        }
    }
    // digit starts: exclusive scan of the global digit histogram
    if (t < 256) {
        const int v = a.counters[kCntHist + (a.shift ? 256 : 0) + t];
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane == 31) s_wsum[warp] = incl;
        s_run[t] = incl - v + excl;  // completed with the earlier warps' sums below
    }
    if (EMIT && warp == 8) {  // offset starts: exclusive scan of the per-offset totals
        const int64_t v = lane < a.k3 ? a.counters[kCntOff + lane] : 0;
        int64_t incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane < a.k3) s_orun[0][lane] = incl - v + excl;
        if (tile == 0) {
            if (lane < a.k3) a.pair_off[lane] = incl - v;
            const int64_t all = __shfl_sync(0xFFFFFFFFu, incl, 31);
            if (lane == 0) a.pair_off[a.k3] = all;
        }
    }
    __syncthreads();
    if (t < 256)
        for (int q = 0; q < warp; ++q) s_run[t] += s_wsum[q];
    __syncthreads();
    bool over = false, bad = false;
#pragma unroll
    for (int r = 0; r < kSwRounds; ++r) {
        const int p = r & 1;
        const bool live = val[r] >= 0;
        const uint32_t d = (key[r] >> a.shift) & 255u;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d : 256u + lane);
        if (live && (peers & lt) == 0) s_cnt[p][warp][d] = __popc(peers);
        const uint32_t m = (EMIT && live) ? mk[r] : 0u;
        uint32_t any = 0;
        if (EMIT) {
            s_pw[p][warp][lane] = 0;
            __syncwarp();
            any = __reduce_or_sync(0xFFFFFFFFu, m);
            for (uint32_t b = any; b; b &= b - 1) {
                const int k = __ffs(b) - 1;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
                if (lane == 0) s_pw[p][warp][k] = __popc(hits);
            }
        }
        __syncthreads();
        int64_t dst = 0;
        bool put = false;
        if (live) {
            int pre = s_run[d] + __popc(peers & lt);
            for (int w = 0; w < warp; ++w) pre += s_cnt[p][w][d];
            dst = pre;
            // totals that disagree with the rows (never for maps the front ends built)
            put = dst >= 0 && dst < a.n;
            if (!put) bad = true;
        }
        if (EMIT && t < a.k3) {  // per offset: exclusive prefix over the warps, and the next round's start
            int run = 0;
            for (int w = 0; w < kSwWarps; ++w) {
                const int c = s_pw[p][w][t];
                s_pw[p][w][t] = run;
                run += c;
            }
            s_orun[p ^ 1][t] = s_orun[p][t] + run;
        }
        __syncthreads();
        if (t < 256) {  // digit t: advance its position and clear this round's counts
            int add = 0;
#pragma unroll
            for (int w = 0; w < kSwWarps; ++w) {
                add += s_cnt[p][w][t];
                s_cnt[p][w][t] = 0;
            }
            s_run[t] += add;
        }
        if (EMIT) {
            for (uint32_t b = any; b; b &= b - 1) {
                const int k = __ffs(b) - 1;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
                if ((m >> k) & 1u) {
                    const int64_t pos = s_orun[p][k] + s_pw[p][warp][k] + __popc(hits & lt);
                    if (pos < a.capacity) {
                        a.pair_in[pos] = k == a.centre ? val[r] : __ldg(a.nbr + int64_t(k) * a.n + val[r]);
                        a.pair_out[pos] = val[r];
                    } else {
                        over = true;
                    }
                }
            }
        }
        if (LAST) {
            if (put) a.perm[dst] = val[r];
            // one atomic per (warp, output tile)
            const uint32_t tl = put ? uint32_t(dst / LAT_TILE_ROWS) : (0x80000000u | lane);
            const unsigned tp = __match_any_sync(0xFFFFFFFFu, tl);
            const uint32_t m_or = __reduce_or_sync(tp, mk[r]);
            if (put && (tp & lt) == 0) atomicOr(a.tile_mask + dst / LAT_TILE_ROWS, m_or);
        } else if (put) {
            a.keys_out[dst] = key[r];
            a.vals_out[dst] = val[r];
            a.masks_out[dst] = mk[r];
        }
    }
    if (over || bad) flag(a.d_status, (over ? LAT_ERR_CAPACITY : 0) | (bad ? LAT_ERR_BAD_MAP : 0));
}

// ----------------------------------------------------------------------------- workspace and host side
struct KmapWs {
    uint32_t *keys;       // grouping key of every row (front end)
    uint32_t *keys_tmp;   // rows after the first sweep: key, row, mask
    int32_t *vals_tmp;
    uint32_t *masks_tmp;
    int32_t *counters;    // kCntWords words, then the look-back words of both sweeps
    unsigned long long *status[2];
    int64_t ntile;
    int64_t zero_words;   // 32-bit words from `counters` on that must be zero before the front end
    size_t total;
};

static KmapWs carve_kmap_ws(void *base, int64_t n_out) {
    KmapWs w{};
    w.ntile = (n_out + kSwTile - 1) / kSwTile;
    Carver cv(base);
    w.keys = cv.take<uint32_t>(size_t(n_out));
    w.keys_tmp = cv.take<uint32_t>(size_t(n_out));
    w.vals_tmp = cv.take<int32_t>(size_t(n_out));
    w.masks_tmp = cv.take<uint32_t>(size_t(n_out));
    w.counters = cv.take<int32_t>(kCntWords);  // kCntWords * 4 is a multiple of 256: status follows directly
    static_assert(kCntWords * 4 % 256 == 0, "counters and look-back words are one contiguous zero region");
    w.status[0] = cv.take<unsigned long long>(size_t(w.ntile) * kSwChains);
    w.status[1] = cv.take<unsigned long long>(size_t(w.ntile) * kSwChains);
    w.zero_words = kCntWords + 2 * 2 * w.ntile * kSwChains;
    w.total = align_up(cv.used, 256);
    return w;
}

// The sweeps of one map whose front end has written nbr, mask, w.keys and the
// global totals: pair lists, perm and tile masks.
static lat_status sweep_map(lat_kmap *map, int k3, const KmapWs &w, int centre, int32_t *d_status, cudaStream_t s) {
    const int64_t n = map->n_out;
    Sweep a{};
    a.keys_in = w.keys;
    a.vals_in = nullptr;
    a.masks_in = map->mask;
    a.n = n;
    a.shift = 0;
    a.counters = w.counters;
    a.which = 0;
    a.status = w.status[0];
    a.nbr = map->nbr;
    a.centre = centre;
    a.k3 = k3;
    a.pair_in = map->pair_in;
    a.pair_out = map->pair_out;
    a.capacity = map->pair_capacity;
    a.pair_off = map->pair_off;
    a.perm = map->perm;
    a.tile_mask = map->tile_mask;
    a.d_status = d_status;
    const dim3 grid(unsigned(w.ntile)), block(kSwThreads);
    if (group_key_bits(k3) <= 8) {
        LAT_CUDA_TRY(launch_pdl(sweep_kernel<true, true>, grid, block, 0, s, a));
        LAT_CUDA_TRY(cudaGetLastError());
        return LAT_OK;
    }
    a.keys_out = w.keys_tmp;
    a.vals_out = w.vals_tmp;
    a.masks_out = w.masks_tmp;
    LAT_CUDA_TRY(launch_pdl(sweep_kernel<true, false>, grid, block, 0, s, a));
    LAT_CUDA_TRY(cudaGetLastError());
    Sweep b = a;
    b.keys_in = w.keys_tmp;
    b.vals_in = w.vals_tmp;
    b.masks_in = w.masks_tmp;
    b.shift = 8;
    b.which = 1;
    b.status = w.status[1];
    LAT_CUDA_TRY(launch_pdl(sweep_kernel<false, true>, grid, block, 0, s, b));
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
    return lat::carve_kmap_ws(nullptr, n_out).total;
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
    const KmapWs need = carve_kmap_ws(nullptr, n_out);
    if (ws_bytes < need.total || (need.total && !ws)) return LAT_ERR_WORKSPACE;
    map->mode = geom->mode;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (n_out == 0) {
        LAT_CUDA_TRY(cudaMemsetAsync(map->pair_off, 0, sizeof(int64_t) * (k3 + 1), s));
        return LAT_OK;
    }
    const KmapWs w = carve_kmap_ws(ws, n_out);
    const int64_t ntiles = (n_out + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS;
    const uint32_t cap_mask = uint32_t(table_bytes / kSlotBytes - 1);
    const SlotGroup *slots = static_cast<const SlotGroup *>(table);
    const int4 *oc = reinterpret_cast<const int4 *>(out_coords);
    FillList f;
    f.add(w.counters, w.zero_words, 0u);
    f.add(map->tile_mask, ntiles, 0u);
    LAT_CUDA_TRY(fill_list(f, s));
    int centre = -1;
    if (geom->mode == LAT_SUBM) {
        SubmGeom g{geom->ksize[0], geom->ksize[1], geom->ksize[2], geom->pad[0], geom->pad[1], geom->pad[2], k3};
        const dim3 grid(unsigned((n_out + kProbeRows - 1) / kProbeRows)), block(32 * g.kx * g.ky);
        if (g.kz == 3)
            LAT_CUDA_TRY(launch_pdl(subm_probe_kernel<3>, grid, block, 0, s, slots, cap_mask, oc, n_out, g, map->nbr,
                                    map->mask, w.keys, w.counters, d_status));
        else if (g.kz == 1)
            LAT_CUDA_TRY(launch_pdl(subm_probe_kernel<1>, grid, block, 0, s, slots, cap_mask, oc, n_out, g, map->nbr,
                                    map->mask, w.keys, w.counters, d_status));
        else
            LAT_CUDA_TRY(launch_pdl(subm_probe_kernel<0>, grid, block, 0, s, slots, cap_mask, oc, n_out, g, map->nbr,
                                    map->mask, w.keys, w.counters, d_status));
        centre = k3 / 2;
    } else {
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
        for (int a = 0; a < 3; ++a) {
            const int d0 = sign * (0 - g.pd[a]), d1 = sign * (g.ks[a] - 1 - g.pd[a]);
            const int dmin = d0 < d1 ? d0 : d1, dmax = d0 < d1 ? d1 : d0;
            g.lo[a] = -32768 - dmin;
            g.hi[a] = 32767 - dmax;
        }
        for (int ix = 0, k = 0; ix < g.ks[0]; ++ix)
            for (int iy = 0; iy < g.ks[1]; ++iy)
                for (int iz = 0; iz < g.ks[2]; ++iz, ++k) {
                    g.off[k][0] = static_cast<signed char>(ix);
                    g.off[k][1] = static_cast<signed char>(iy);
                    g.off[k][2] = static_cast<signed char>(iz);
                    const long long dx = sign * (ix - g.pd[0]), dy = sign * (iy - g.pd[1]),
                                    dz = sign * (iz - g.pd[2]);
                    g.delta[k] = dx * (1ll << 32) + dy * (1ll << 16) + dz;
                }
        const int nblk = int((n_out + kQueryThreads - 1) / kQueryThreads);
        LAT_CUDA_TRY(launch_pdl(kmap_probe_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, slots, cap_mask, oc, n_out,
                                n_in, g, map->nbr, map->mask, w.keys, w.counters, d_status));
    }
    LAT_CUDA_TRY(cudaGetLastError());
    return sweep_map(map, k3, w, centre, d_status, s);
}

extern "C" size_t lat_kmap_from_parent_ws_bytes(int64_t n_fine, int64_t n_coarse, int32_t k3) {
    if (n_fine < 0 || n_coarse < 0 || n_fine >= (int64_t(1) << 31) || n_coarse >= (int64_t(1) << 31) || k3 < 1 ||
        k3 > 32)
        return 0;
    // the strided map's workspace, then the transposed map's
    return lat::carve_kmap_ws(nullptr, n_coarse).total + lat::carve_kmap_ws(nullptr, n_fine).total;
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
    const KmapWs w_down = carve_kmap_ws(ws, n_coarse);
    const KmapWs w_up = carve_kmap_ws(static_cast<char *>(ws) + w_down.total, n_fine);
    // every initialisation both maps need, in one launch: the strided map's
    // table (-1) and masks (0, both filled by the parent scatter), and each
    // map's counters, look-back words and tile masks
    FillList f;
    if (down && n_coarse > 0) {
        f.add(down->nbr, int64_t(k3) * n_coarse, ~0u);
        f.add(down->mask, n_coarse, 0u);
        f.add(w_down.counters, w_down.zero_words, 0u);
        f.add(down->tile_mask, (n_coarse + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS, 0u);
    }
    if (up && n_fine > 0) {
        f.add(w_up.counters, w_up.zero_words, 0u);
        f.add(up->tile_mask, (n_fine + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS, 0u);
    }
    LAT_CUDA_TRY(fill_list(f, s));
    if (n_fine > 0) {
        LAT_CUDA_TRY(launch_pdl(parent_maps_kernel, dim3(unsigned((n_fine + 255) / 256)), dim3(256), 0, s,
                                reinterpret_cast<const int4 *>(fine_coords), parent, n_fine, n_coarse, geom->stride[0],
                                geom->stride[1], geom->stride[2], k3, up ? up->nbr : nullptr, up ? up->mask : nullptr,
                                up ? w_up.keys : nullptr, w_up.counters, down ? down->nbr : nullptr,
                                down ? down->mask : nullptr, d_status));
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
        const cudaStream_t ms = (side && map == up) ? side->side : main_s;
        if (map->n_out == 0) {
            LAT_CUDA_TRY(cudaMemsetAsync(map->pair_off, 0, sizeof(int64_t) * (k3 + 1), ms));
            continue;
        }
        const KmapWs &w = map == down ? w_down : w_up;
        if (map == down) {
            const int nblk = int((map->n_out + kQueryThreads - 1) / kQueryThreads);
            LAT_CUDA_TRY(launch_pdl(kmap_count_kernel, dim3(nblk), dim3(kQueryThreads), 0, ms, map->mask, map->n_out,
                                    k3, w.keys, w.counters));
            LAT_CUDA_TRY(cudaGetLastError());
        }
        const lat_status st = sweep_map(map, k3, w, -1, d_status, ms);
        if (st != LAT_OK) return st;
    }
    if (side) LAT_CUDA_TRY(side_join(*side, main_s));
    return LAT_OK;
}
