// Kernel-map construction / coordinate query (lat_kmap_ws_bytes, lat_kmap_query,
// lat_kmap_from_parent).
//
// Torch Lattice docs, "Migrating from TorchSparse": kernel-map construction
// and coordinate query are CUDA kernels of the library ("What remains
// familiar", "Sparse tensor expectations"), and the support semantics come
// from the "Convolution mapping" table.  Pipeline of one map (all on
// `stream`):
//   0. fill:   zeroes the per-tile counts and the tile masks (submanifold maps:
//              also -1 in the offsets above the centre, centre bit in every mask).
//   1. front end: nbr (offset-major), the neighbour mask and the grouping key
//              of every output row, and per tile of kScTile rows the counts of
//              the key's low byte and of the pairs of every offset.
//                submanifold: kmap_probe_col_kernel (one thread per (row,
//                                   z-column of offsets below the centre; one or
//                                   two z-brick group scans per column), each hit
//                                   mirrored into the upper half; columns of more
//                                   than kColMaxCells cells: kmap_probe_sym_kernel,
//                                   one thread per (row, offset)) + kmap_count_kernel
//                strided/transposed: kmap_probe_kernel (a row per thread)
//                maps from parents: parent_maps_kernel (+ kmap_count_kernel)
//   2. row scan: one block per digit (and per offset) turns its per-tile
//              counts into tile starts and a total.
//   3. scatter 1: the pair lists (grouped by offset, output rows ascending)
//              and the first stable radix pass of the rows by the key's low
//              byte, counting the high byte per output tile.
//   4. row scan, 5. scatter 2: the second pass (high byte) -> perm and the
//              tile masks.  With K^3 <= 8 the key is the mask itself (one
//              byte) and scatter 1 writes perm and the tile masks directly.
// Ranks inside a tile keep row order, so the sort is stable and every output
// is deterministic.
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

// ----------------------------------------------------------------------------- per-tile counts
// The scatter passes work on tiles of kScTile rows.  Their first pass needs,
// per tile, the count of every value of the key's low byte and of the pairs
// of every offset: chain c (c < 256: digit c, 256 + k: offset k) of tile b at
// cnt[c * ntile + b].  Front-end blocks cover whole rows of one tile and add
// their block's counts with one atomic per nonzero value.
constexpr int kScThreads = 256;
constexpr int kScWarps = kScThreads / 32;
constexpr int kScRounds = 2;
constexpr int kScTile = kScThreads * kScRounds;  // rows per scatter tile
constexpr int kChains = 256 + 32;

// Shared-memory tallies of one block (s_h: the key's low byte, s_o: pairs per offset).
struct Tally {
    int *s_h;  // [256]
    int *s_o;  // [32]
};

// Counts one row per lane into the block's tallies; every lane of the warp calls it.
__device__ __forceinline__ void tally_row(const Tally &ty, uint32_t key, uint32_t m, bool live) {
    const int lane = threadIdx.x & 31;
    const uint32_t d0 = key & 255u;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d0 : 256u + lane);
    if (live && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&ty.s_h[d0], int(__popc(peers)));
    const uint32_t mm = live ? m : 0u;
    for (uint32_t any = __reduce_or_sync(0xFFFFFFFFu, mm); any; any &= any - 1) {
        const int k = __ffs(any) - 1;
        const unsigned hits = __ballot_sync(0xFFFFFFFFu, (mm >> k) & 1u);
        if (lane == 0) atomicAdd(&ty.s_o[k], int(__popc(hits)));
    }
}

__device__ __forceinline__ void tally_clear(const Tally &ty) {
    for (int i = threadIdx.x; i < 256 + 32; i += blockDim.x) (i < 256 ? ty.s_h[i] : ty.s_o[i - 256]) = 0;
}

// Adds the block's tallies to its tile's counts (after a __syncthreads()).
__device__ __forceinline__ void tally_flush(const Tally &ty, int k3, int32_t *cnt, int ntile, int64_t first_row) {
    const int64_t tile = first_row / kScTile;
    for (int i = threadIdx.x; i < 256 + k3; i += blockDim.x) {
        const int v = i < 256 ? ty.s_h[i] : ty.s_o[i - 256];
        if (v) atomicAdd(cnt + int64_t(i) * ntile + tile, v);
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

__device__ __forceinline__ bool query_coord(const Geom &g, const int4 &c, int ix, int iy, int iz, uint64_t &key);

// ----------------------------------------------------------------------------- submanifold front end
// Submanifold map: one thread per (offset k below the centre, row j);
// blockIdx.y is the offset, so a warp probes one offset for 32 consecutive rows
// (coalesced coordinate loads and nbr stores, a uniform key delta).  A probe
// reads its home group's 4 keys with two 16-byte loads and walks on to the next
// group only when all 4 slots hold other keys (bounded by the probe window).
// A hit at row r also writes the mirrored entry nbr[k3-1-k][r] = j (the
// relation is symmetric) and ORs both bits into the masks.  The fill before
// it set the offsets above the centre to -1 and every mask to the centre bit;
// the threads of offset 0 also write the centre column (every row is its own
// centre neighbour).  Far fewer instructions per lookup than looping over the
// offsets inside one thread, and about 30 registers, so every SM runs its full
// complement of warps.
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
    if (k == 0) nbr[int64_t(g.k3 / 2) * n_out + j] = int32_t(j);
    if (r >= 0) {
        const int km = g.k3 - 1 - k;
        nbr[int64_t(km) * n_out + r] = int32_t(j);
        atomicOr(mask + j, 1u << k);
        atomicOr(mask + r, 1u << km);
    }
}

// Column form of the submanifold front end.  The offsets below the centre
// that share (dx, dy) form a run of consecutive z offsets -- a "column" -- and
// the hash places the 4 cells of a z-brick (z = 4m..4m+3 of one (b, x, y))
// in one home group, so a column of up to kColMaxCells cells touches at most
// two bricks: one thread per (row, column) looks up those one or two bricks
// (a group's 4 keys, two 16-byte loads each) instead of probing every cell,
// and loads a row only for the cells present.  Outputs, mirror writes and
// mask bits are exactly those of kmap_probe_sym_kernel.
constexpr int kColMax = 16;
constexpr int kColMaxCells = 5;
struct Col {
    long long delta;  // key delta of the column's first cell
    int kbase;        // offset index of that cell; the column's cells are kbase, kbase + 1, ...
    int n;            // cells, 1..kColMaxCells
};
struct Cols {
    Col c[kColMax];
    int count;
};

// Scans the 4 keys of group gi for brick key B (halves bh, bl; bl's low two
// bits clear): for each key B + d found, sets bit d of occ and puts tag | slot
// (3 bits) at bits 3d of sel.  Returns whether the group has an empty slot.
__device__ __forceinline__ bool brick_scan(const SlotGroup *groups, uint32_t gi, uint32_t bh, uint32_t bl,
                                           uint32_t tag, uint32_t &occ, uint32_t &sel) {
    const uint4 *gp = reinterpret_cast<const uint4 *>(groups + gi);
    const uint4 a = __ldg(gp), b = __ldg(gp + 1);  // keys 0, 1 and 2, 3 as (lo, hi) word pairs
    const uint32_t lo[kGroupSlots] = {a.x, a.z, b.x, b.z};
    const uint32_t hi[kGroupSlots] = {a.y, a.w, b.y, b.w};
    bool empty = false;
#pragma unroll
    for (int i = 0; i < kGroupSlots; ++i) {
        const uint32_t d = lo[i] - bl;  // < 4 only for a key of the brick (the high halves must match too)
        if (hi[i] == bh && d < 4u) {
            occ |= 1u << d;
            sel |= (tag | uint32_t(i)) << (3u * d);
        }
        empty |= hi[i] == 0xFFFFFFFFu;  // no packed key has an all-ones high half
    }
    return empty;
}

// The present z positions of brick key B (low two bits clear): bit d of occ
// set if key B + d is in the table; bits 3d of sel give its slot (2 bits) and
// whether it sits in the home group grp (0) or the next group (4).  Linear
// probing fills a group's slots in order, so a group with an empty slot, or
// the 4 cells of the brick found, ends the scan; returns false if the next
// group is full too and the brick incomplete (the caller then probes cell by
// cell).
__device__ __forceinline__ bool brick_lookup(const SlotGroup *groups, uint32_t cap_mask, uint64_t B, uint32_t &occ,
                                             uint32_t &sel, uint32_t &grp) {
    grp = probe_start(B, cap_mask) / kGroupSlots;
    const uint32_t bh = uint32_t(B >> 32), bl = uint32_t(B);
    occ = 0;
    sel = 0;
    if (brick_scan(groups, grp, bh, bl, 0u, occ, sel) || occ == 0xFu) return true;
    return brick_scan(groups, (grp + 1) & (cap_mask / kGroupSlots), bh, bl, 4u, occ, sel) || occ == 0xFu;
}

// Row of key `key` (linear probing from its home group), -1 if absent.
__device__ __forceinline__ int probe_row(const SlotGroup *groups, uint32_t cap_mask, uint64_t key) {
    const int slot = probe_one(groups, cap_mask, key);
    return slot < 0 ? -1 : int(__ldg(&groups[slot / kGroupSlots].row[slot % kGroupSlots]));
}

// One thread per (row j, column blockIdx.y).  Rows whose offsets could leave
// the key fields, and columns whose brick lookup ends in a full group, take
// the cells one at a time.  Threads of column 0 also write the centre column.
__global__ void __launch_bounds__(kQueryThreads)
kmap_probe_col_kernel(const SlotGroup *__restrict__ groups, uint32_t cap_mask, const int4 *__restrict__ out_coords,
                      int64_t n_out, Geom g, Cols cols, int32_t *__restrict__ nbr, uint32_t *__restrict__ mask,
                      int32_t *d_status) {
    pdl_enter();
    const Col col = cols.c[blockIdx.y];
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    if (j >= n_out) return;
    const int4 c = __ldg(out_coords + j);
    if (blockIdx.y == 0) nbr[int64_t(g.k3 / 2) * n_out + j] = int32_t(j);
    int rr[kColMaxCells];
    uint64_t key = 0;
    bool fast = g.shift && c.y >= g.lo[0] && c.y <= g.hi[0] && c.z >= g.lo[1] && c.z <= g.hi[1] &&
                c.w >= g.lo[2] && c.w <= g.hi[2] && pack_key(c.x, c.y, c.z, c.w, key);
    if (fast) {
        const uint64_t kc = key + uint64_t(col.delta);  // the column's first cell
        const uint64_t b1 = kc & ~uint64_t(3);
        const uint32_t p0 = uint32_t(kc) & 3u;          // its z position within brick b1
        uint32_t occ, sel, grp, occ2 = 0, sel2 = 0, grp2 = 0;
        fast = brick_lookup(groups, cap_mask, b1, occ, sel, grp);
        if (p0 + uint32_t(col.n) > 4u) fast &= brick_lookup(groups, cap_mask, b1 + 4, occ2, sel2, grp2);
        occ |= occ2 << 4;
        const uint32_t gmask = cap_mask / kGroupSlots;
#pragma unroll
        for (int t = 0; t < kColMaxCells; ++t) {
            const uint32_t pos = p0 + uint32_t(t);
            rr[t] = -1;
            if (t < col.n && fast && ((occ >> pos) & 1u)) {
                const uint32_t code = pos < 4u ? (sel >> (3u * pos)) : (sel2 >> (3u * (pos - 4u)));
                const uint32_t gi = ((pos < 4u ? grp : grp2) + (code >> 2 & 1u)) & gmask;
                rr[t] = int(__ldg(&groups[gi].row[code & 3u]));
            }
        }
    }
    if (!fast) {
#pragma unroll
        for (int t = 0; t < kColMaxCells; ++t) {
            rr[t] = -1;
            if (t < col.n) {
                const int k = col.kbase + t;
                uint64_t kk;
                if (query_coord(g, c, g.off[k][0], g.off[k][1], g.off[k][2], kk)) rr[t] = probe_row(groups, cap_mask, kk);
            }
        }
    }
    uint32_t jbits = 0;
#pragma unroll
    for (int t = 0; t < kColMaxCells; ++t) {
        if (t >= col.n) break;
        const int k = col.kbase + t;
        int r = rr[t];
        if (r >= n_out) {
            flag(d_status, LAT_ERR_BAD_MAP);
            r = -1;
        }
        nbr[int64_t(k) * n_out + j] = r;
        if (r >= 0) {
            const int km = g.k3 - 1 - k;
            nbr[int64_t(km) * n_out + r] = int32_t(j);
            atomicOr(mask + r, 1u << km);
            jbits |= 1u << k;
        }
    }
    if (jbits) atomicOr(mask + j, jbits);
}

// The columns of a submanifold geometry's lower half (offsets below the
// centre), in offset order; false if a column has more than kColMaxCells
// cells (the per-offset kernel then runs).
static bool subm_columns(const Geom &g, Cols &cols) {
    const int centre = g.k3 / 2;
    cols.count = 0;
    for (int k = 0; k < centre;) {
        const int ix = g.off[k][0], iy = g.off[k][1];
        int n = 0;
        while (k + n < centre && g.off[k + n][0] == ix && g.off[k + n][1] == iy) ++n;
        if (n > kColMaxCells || cols.count == kColMax) return false;
        Col &cl = cols.c[cols.count++];
        cl.delta = g.delta[k];
        cl.kbase = k;
        cl.n = n;
        k += n;
    }
    return cols.count > 0;
}

// A submanifold map with a single offset (1x1x1): every row is its own neighbour.
__global__ void __launch_bounds__(kQueryThreads) kmap_centre_kernel(int64_t n_out, int32_t *__restrict__ nbr) {
    pdl_enter();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    if (j < n_out) nbr[j] = int32_t(j);
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
                  uint32_t *__restrict__ keys, int32_t *__restrict__ cnt, int ntile, int32_t *d_status) {
    pdl_enter();
    __shared__ int s_h[256], s_o[32];
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
    tally_row(ty, key, m, live);
    __syncthreads();
    tally_flush(ty, g.k3, cnt, ntile, blockIdx.x * int64_t(kQueryThreads));
}

// Grouping keys and global totals from final masks (the strided map of a
// ksize == stride convolution, whose masks the parent scatter builds).
__global__ void __launch_bounds__(kQueryThreads)
kmap_count_kernel(const uint32_t *__restrict__ mask, int64_t n_out, int k3, uint32_t *__restrict__ keys,
                  int32_t *__restrict__ cnt, int ntile) {
    pdl_enter();
    __shared__ int s_h[256], s_o[32];
    const Tally ty{s_h, s_o};
    tally_clear(ty);
    __syncthreads();
    const int64_t j = blockIdx.x * int64_t(kQueryThreads) + threadIdx.x;
    const bool live = j < n_out;
    const uint32_t m = live ? __ldg(mask + j) : 0u;
    const uint32_t key = group_key(m, k3);
    if (live) keys[j] = key;
    tally_row(ty, key, m, live);
    __syncthreads();
    tally_flush(ty, k3, cnt, ntile, blockIdx.x * int64_t(kQueryThreads));
}

// Kernel size == stride, no padding: fine row i lies in exactly one coarse window,
// parent[i], at offset k(i) = its position inside the window (floor modulo the
// stride per axis).  Writes the transposed map's rows directly (one neighbour
// per fine row), with their grouping keys and totals, and scatters the strided
// map's entries (its table must hold -1 and its masks 0 beforehand).
__global__ void __launch_bounds__(256)
parent_maps_kernel(const int4 *__restrict__ fine, const int32_t *__restrict__ parent, int64_t n_fine,
                   int64_t n_coarse, int s0, int s1, int s2, int k3, int32_t *__restrict__ up_nbr,
                   uint32_t *__restrict__ up_mask, uint32_t *__restrict__ up_keys, int32_t *__restrict__ up_cnt,
                   int up_ntile, int32_t *__restrict__ down_nbr, uint32_t *__restrict__ down_mask, int32_t *d_status) {
    pdl_enter();
    __shared__ int s_h[256], s_o[32];
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
        tally_row(ty, key, m, live);
        __syncthreads();
        tally_flush(ty, k3, up_cnt, up_ntile, blockIdx.x * int64_t(blockDim.x));
    }
}

// ----------------------------------------------------------------------------- row scan and scatter passes
// Block c: exclusive scan, in place, of chain c's per-tile counts
// cnt[c * ntile + 0 .. ntile) (the first row of each tile), and the chain's
// total into totals[c].  1024 threads: one pass covers 1024 tiles (512k rows).
constexpr int kRowScanThreads = 1024;
__global__ void __launch_bounds__(kRowScanThreads)
row_scan_kernel(int32_t *__restrict__ cnt, int ntile, int32_t *__restrict__ totals) {
    pdl_enter();
    constexpr int kWarps = kRowScanThreads / 32;
    __shared__ int s_warp[kWarps];  // per warp: its sum, then the sum of the warps before it
    __shared__ int s_total;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    int32_t *row = cnt + int64_t(blockIdx.x) * ntile;
    int carry = 0;
    for (int base = 0; base < ntile; base += kRowScanThreads) {
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
        if (w == 0) {
            const int x = s_warp[lane];
            int wi = x;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, wi, d);
                if (lane >= d) wi += o;
            }
            s_warp[lane] = wi - x;
        }
        __syncthreads();
        const int before = s_warp[w];
        if (i < ntile) row[i] = carry + before + incl - v;
        if (t == kRowScanThreads - 1) s_total = before + incl;
        __syncthreads();
        carry += s_total;
        __syncthreads();
    }
    if (t == 0) totals[blockIdx.x] = carry;
}

struct Scatter {
    const uint32_t *keys_in;   // key of each input position
    const int32_t *vals_in;    // output row of each input position; nullptr = the position itself
    const uint32_t *masks_in;  // neighbour mask of each input position
    int64_t n;
    int shift;                 // this pass's digit: (key >> shift) & 255
    const int32_t *cnt;        // chains x tiles: each tile's first position among its chain (row-scanned)
    const int32_t *totals;     // per chain: 256 digits, then (EMIT) k3 offsets
    int ntile;
    // pair emission (first pass)
    const int32_t *nbr;
    int centre;  // offset whose neighbour of row j is j itself (submanifold), else -1
    int k3;
    int32_t *pair_in, *pair_out;
    int64_t capacity;
    int64_t *pair_off;
    // outputs: to the second pass (with its per-tile counts), or perm and the tile masks
    uint32_t *keys_out;
    int32_t *vals_out;
    uint32_t *masks_out;
    int32_t *cnt_next;    // [256][ntile], zero at launch
    int32_t *perm;
    uint32_t *tile_mask;  // zero at launch
    int32_t *d_status;
};

// One tile of one stable radix pass.  EMIT: also write the pair lists (first
// pass, rows in input order).  LAST: write perm and OR each row's mask into
// its LAT_TILE_ROWS output tile; otherwise hand (key, row, mask) to the next
// pass at the sorted position and count the next digit per output tile.
// Position of a row: its digit's start (exclusive scan of the digit totals)
// + the tile's start among that digit (row scan) + the row's rank among the
// tile's rows of that digit (warp match; per round, one thread per digit turns
// the per-warp counts into per-warp starts with its loads issued together).
// Pair positions likewise per offset; the pairs' neighbour rows are loaded
// kEmitBatch at a time before any of them is stored.
constexpr int kEmitBatch = 4;

template <bool EMIT, bool LAST>
__global__ void __launch_bounds__(kScThreads) scatter_kernel(Scatter a) {
    pdl_wait();
    __shared__ int s_cnt[kScWarps][256];        // this round: per-warp rows of each digit
    __shared__ int s_pre[kScWarps][256];        // this round: first position of each (warp, digit)
    __shared__ int s_run[256];                  // next position of each digit
    __shared__ int s_pw[kScWarps][32];          // this round: per-warp pairs of each offset
    __shared__ unsigned s_ball[kScWarps][32];   // this round: per warp, the lanes with a pair at each offset
    __shared__ long long s_pwx[kScWarps][32];   // this round: first pair position of each (warp, offset)
    __shared__ long long s_orun[32];            // next pair position of each offset
    __shared__ long long s_cbase;               // first pair of the centre offset (submanifold maps)
    __shared__ int s_wsum[kScWarps];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const int tile = blockIdx.x;
    uint32_t key[kScRounds], mk[kScRounds];
    int32_t val[kScRounds];
#pragma unroll
    for (int r = 0; r < kScRounds; ++r) {
        const int64_t e = int64_t(tile) * kScTile + r * kScThreads + t;
        key[r] = 0;
        mk[r] = 0;
        val[r] = -1;
        if (e < a.n) {
            key[r] = __ldg(a.keys_in + e);
            val[r] = a.vals_in ? __ldg(a.vals_in + e) : int32_t(e);
            if (EMIT || LAST) mk[r] = __ldg(a.masks_in + e);
        }
    }
    for (int i = t; i < kScWarps * 256; i += kScThreads) (&s_cnt[0][0])[i] = 0;
    {  // digit starts: exclusive scan of the digit totals, plus this tile's start
        const int v = __ldg(a.totals + t);
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane == 31) s_wsum[warp] = incl;
        s_run[t] = incl - v + __ldg(a.cnt + int64_t(t) * a.ntile + tile);  // + the earlier warps' sums below
    }
    if (EMIT && warp == 0) {  // offset starts: exclusive scan of the offset totals, plus this tile's start
        const int64_t v = lane < a.k3 ? __ldg(a.totals + 256 + lane) : 0;
        int64_t incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane < a.k3) s_orun[lane] = incl - v + __ldg(a.cnt + int64_t(256 + lane) * a.ntile + tile);
        if (a.centre >= 0 && lane == a.centre) s_cbase = incl - v;
        if (tile == 0) {
            if (lane < a.k3) a.pair_off[lane] = incl - v;
            const int64_t all = __shfl_sync(0xFFFFFFFFu, incl, 31);
            if (lane == 0) a.pair_off[a.k3] = all;
        }
    }
    pdl_trigger();
    __syncthreads();
    for (int q = 0; q < warp; ++q) s_run[t] += s_wsum[q];
    bool over = false, bad = false;
#pragma unroll
    for (int r = 0; r < kScRounds; ++r) {
        const bool live = val[r] >= 0;
        const uint32_t d = (key[r] >> a.shift) & 255u;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, live ? d : 256u + lane);
        if (live && (peers & lt) == 0) s_cnt[warp][d] = __popc(peers);
        // the centre pair of every row (j, j) sits at a fixed position; the
        // other offsets are counted per warp, with the lanes that have them
        const uint32_t cbit = a.centre >= 0 ? 1u << a.centre : 0u;
        const uint32_t m = (EMIT && live) ? mk[r] & ~cbit : 0u;
        if (EMIT) {
            s_pw[warp][lane] = 0;
            __syncwarp();
            for (uint32_t b = __reduce_or_sync(0xFFFFFFFFu, m); b; b &= b - 1) {
                const int k = __ffs(b) - 1;
                const unsigned hits = __ballot_sync(0xFFFFFFFFu, (m >> k) & 1u);
                if (lane == 0) {
                    s_pw[warp][k] = __popc(hits);
                    s_ball[warp][k] = hits;
                }
            }
        }
        __syncthreads();
        {  // digit t: first position of each warp's rows, counts cleared, start advanced
            int c[kScWarps];
#pragma unroll
            for (int w = 0; w < kScWarps; ++w) c[w] = s_cnt[w][t];
            int run = s_run[t];
#pragma unroll
            for (int w = 0; w < kScWarps; ++w) {
                s_pre[w][t] = run;
                run += c[w];
                s_cnt[w][t] = 0;
            }
            s_run[t] = run;
        }
        if (EMIT && t < a.k3) {  // offset t: the same for the pairs
            int c[kScWarps];
#pragma unroll
            for (int w = 0; w < kScWarps; ++w) c[w] = s_pw[w][t];
            long long run = s_orun[t];
#pragma unroll
            for (int w = 0; w < kScWarps; ++w) {
                s_pwx[w][t] = run;
                run += c[w];
            }
            s_orun[t] = run;
        }
        __syncthreads();
        int64_t dst = 0;
        bool put = false;
        if (live) {
            dst = s_pre[warp][d] + __popc(peers & lt);
            // counts that disagree with the rows (never for maps the front ends built)
            put = dst >= 0 && dst < a.n;
            if (!put) bad = true;
        }
        if (EMIT) {
            if (live && (mk[r] & cbit)) {  // centre pair: every row of a submanifold map has it
                const int64_t pos = s_cbase + val[r];
                if (pos < a.capacity) {
                    a.pair_in[pos] = val[r];
                    a.pair_out[pos] = val[r];
                } else {
                    over = true;
                }
            }
            // this lane's other pairs, kEmitBatch neighbour loads in flight at a time
            for (uint32_t b = m; b;) {
                int kk[kEmitBatch], vv[kEmitBatch];
                int64_t pp[kEmitBatch];
#pragma unroll
                for (int q = 0; q < kEmitBatch; ++q) {
                    kk[q] = -1;
                    if (b) {
                        const int k = __ffs(b) - 1;
                        b &= b - 1;
                        kk[q] = k;
                        pp[q] = s_pwx[warp][k] + __popc(s_ball[warp][k] & lt);
                        vv[q] = __ldg(a.nbr + int64_t(k) * a.n + val[r]);
                    }
                }
#pragma unroll
                for (int q = 0; q < kEmitBatch; ++q) {
                    if (kk[q] < 0) continue;
                    if (pp[q] < a.capacity) {
                        a.pair_in[pp[q]] = vv[q];
                        a.pair_out[pp[q]] = val[r];
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
        } else {
            if (put) {
                a.keys_out[dst] = key[r];
                a.vals_out[dst] = val[r];
                a.masks_out[dst] = mk[r];
            }
            // the next pass's digit per output tile: one atomic per (warp, digit, tile);
            // output tile < 2^31 / kScTile <= 2^22, digit < 2^8: the tag fits in 30 bits
            const uint32_t d2 = (key[r] >> (a.shift + 8)) & 255u;
            const uint32_t tag = put ? ((d2 << 22) | uint32_t(dst / kScTile)) : (0x80000000u | lane);
            const unsigned p2 = __match_any_sync(0xFFFFFFFFu, tag);
            if (put && (p2 & lt) == 0) atomicAdd(a.cnt_next + int64_t(d2) * a.ntile + dst / kScTile, int(__popc(p2)));
        }
    }
    if (over || bad) flag(a.d_status, (over ? LAT_ERR_CAPACITY : 0) | (bad ? LAT_ERR_BAD_MAP : 0));
}

// ----------------------------------------------------------------------------- workspace and host side
struct KmapWs {
    uint32_t *keys;       // grouping key of every row (front end)
    uint32_t *keys_tmp;   // rows after the first pass: key, row, mask
    int32_t *vals_tmp;
    uint32_t *masks_tmp;
    int32_t *cnt1;        // [256 + 32][ntile] counts of the first pass (digits, then offsets)
    int32_t *cnt2;        // [256][ntile] counts of the second pass
    int32_t *tot1, *tot2;
    int ntile;
    int64_t zero_words;   // cnt1 and cnt2 are one contiguous region that must be zero before the front end
    size_t total;
};

static KmapWs carve_kmap_ws(void *base, int64_t n_out) {
    KmapWs w{};
    w.ntile = int((n_out + kScTile - 1) / kScTile);
    Carver cv(base);
    w.keys = cv.take<uint32_t>(size_t(n_out));
    w.keys_tmp = cv.take<uint32_t>(size_t(n_out));
    w.vals_tmp = cv.take<int32_t>(size_t(n_out));
    w.masks_tmp = cv.take<uint32_t>(size_t(n_out));
    w.cnt1 = cv.take<int32_t>(size_t(kChains + 256) * w.ntile);
    w.cnt2 = w.cnt1 ? w.cnt1 + size_t(kChains) * w.ntile : nullptr;
    w.zero_words = int64_t(kChains + 256) * w.ntile;
    w.tot1 = cv.take<int32_t>(kChains);
    w.tot2 = cv.take<int32_t>(256);
    w.total = align_up(cv.used, 256);
    return w;
}

// The passes of one map whose front end has written nbr, mask, w.keys and the
// first pass's per-tile counts: pair lists, perm and tile masks.
static lat_status finish_map(lat_kmap *map, int k3, const KmapWs &w, int centre, int32_t *d_status, cudaStream_t s) {
    Scatter a{};
    a.keys_in = w.keys;
    a.vals_in = nullptr;
    a.masks_in = map->mask;
    a.n = map->n_out;
    a.shift = 0;
    a.cnt = w.cnt1;
    a.totals = w.tot1;
    a.ntile = w.ntile;
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
    const dim3 grid(unsigned(w.ntile)), block(kScThreads);
    LAT_CUDA_TRY(launch_pdl(row_scan_kernel, dim3(256 + k3), dim3(kRowScanThreads), 0, s, w.cnt1, w.ntile, w.tot1));
    LAT_CUDA_TRY(cudaGetLastError());
    if (group_key_bits(k3) <= 8) {
        LAT_CUDA_TRY(launch_pdl(scatter_kernel<true, true>, grid, block, 0, s, a));
        LAT_CUDA_TRY(cudaGetLastError());
        return LAT_OK;
    }
    a.keys_out = w.keys_tmp;
    a.vals_out = w.vals_tmp;
    a.masks_out = w.masks_tmp;
    a.cnt_next = w.cnt2;
    LAT_CUDA_TRY(launch_pdl(scatter_kernel<true, false>, grid, block, 0, s, a));
    LAT_CUDA_TRY(cudaGetLastError());
    LAT_CUDA_TRY(launch_pdl(row_scan_kernel, dim3(256), dim3(kRowScanThreads), 0, s, w.cnt2, w.ntile, w.tot2));
    LAT_CUDA_TRY(cudaGetLastError());
    Scatter b = a;
    b.keys_in = w.keys_tmp;
    b.vals_in = w.vals_tmp;
    b.masks_in = w.masks_tmp;
    b.shift = 8;
    b.cnt = w.cnt2;
    b.totals = w.tot2;
    LAT_CUDA_TRY(launch_pdl(scatter_kernel<false, true>, grid, block, 0, s, b));
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
                const long long dx = sign * (ix - g.pd[0]), dy = sign * (iy - g.pd[1]), dz = sign * (iz - g.pd[2]);
                g.delta[k] = dx * (1ll << 32) + dy * (1ll << 16) + dz;
            }
    const int nblk = int((n_out + kQueryThreads - 1) / kQueryThreads);
    int centre = -1;
    if (geom->mode == LAT_SUBM) {
        centre = k3 / 2;
        FillList f;
        f.add(w.cnt1, w.zero_words, 0u);
        f.add(map->tile_mask, ntiles, 0u);
        f.add(map->nbr + int64_t(centre + 1) * n_out, int64_t(k3 - 1 - centre) * n_out, ~0u);  // filled by mirrors
        f.add(map->mask, n_out, 1u << centre);
        LAT_CUDA_TRY(fill_list(f, s));
        Cols cols;
        if (centre > 0 && subm_columns(g, cols)) {
            LAT_CUDA_TRY(launch_pdl(kmap_probe_col_kernel, dim3(unsigned(nblk), unsigned(cols.count)),
                                    dim3(kQueryThreads), 0, s, slots, cap_mask, oc, n_out, g, cols, map->nbr, map->mask,
                                    d_status));
        } else if (centre > 0) {
            LAT_CUDA_TRY(launch_pdl(kmap_probe_sym_kernel, dim3(unsigned(nblk), unsigned(centre)), dim3(kQueryThreads),
                                    0, s, slots, cap_mask, oc, n_out, g, map->nbr, map->mask, d_status));
        } else {  // 1x1x1: the centre column alone
            LAT_CUDA_TRY(launch_pdl(kmap_centre_kernel, dim3(unsigned(nblk)), dim3(kQueryThreads), 0, s, n_out,
                                    map->nbr));
        }
        LAT_CUDA_TRY(cudaGetLastError());
        LAT_CUDA_TRY(launch_pdl(kmap_count_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, map->mask, n_out, k3, w.keys,
                                w.cnt1, w.ntile));
    } else {
        FillList f;
        f.add(w.cnt1, w.zero_words, 0u);
        f.add(map->tile_mask, ntiles, 0u);
        LAT_CUDA_TRY(fill_list(f, s));
        LAT_CUDA_TRY(launch_pdl(kmap_probe_kernel, dim3(nblk), dim3(kQueryThreads), 0, s, slots, cap_mask, oc, n_out,
                                n_in, g, map->nbr, map->mask, w.keys, w.cnt1, w.ntile, d_status));
    }
    LAT_CUDA_TRY(cudaGetLastError());
    return finish_map(map, k3, w, centre, d_status, s);
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
    // map's per-tile counts and tile masks
    FillList f;
    if (down && n_coarse > 0) {
        f.add(down->nbr, int64_t(k3) * n_coarse, ~0u);
        f.add(down->mask, n_coarse, 0u);
        f.add(w_down.cnt1, w_down.zero_words, 0u);
        f.add(down->tile_mask, (n_coarse + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS, 0u);
    }
    if (up && n_fine > 0) {
        f.add(w_up.cnt1, w_up.zero_words, 0u);
        f.add(up->tile_mask, (n_fine + LAT_TILE_ROWS - 1) / LAT_TILE_ROWS, 0u);
    }
    LAT_CUDA_TRY(fill_list(f, s));
    if (n_fine > 0) {
        LAT_CUDA_TRY(launch_pdl(parent_maps_kernel, dim3(unsigned((n_fine + 255) / 256)), dim3(256), 0, s,
                                reinterpret_cast<const int4 *>(fine_coords), parent, n_fine, n_coarse, geom->stride[0],
                                geom->stride[1], geom->stride[2], k3, up ? up->nbr : nullptr, up ? up->mask : nullptr,
                                up ? w_up.keys : nullptr, w_up.cnt1, w_up.ntile, down ? down->nbr : nullptr,
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
                                    k3, w.keys, w.cnt1, w.ntile));
            LAT_CUDA_TRY(cudaGetLastError());
        }
        const lat_status st = finish_map(map, k3, w, -1, d_status, ms);
        if (st != LAT_OK) return st;
    }
    if (side) LAT_CUDA_TRY(side_join(*side, main_s));
    return LAT_OK;
}
