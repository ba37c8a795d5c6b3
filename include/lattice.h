/*
 * lattice.h -- C ABI of the B200 sparse-convolution library (liblattice.so).
 *
 * Sparse convolution over coordinate-indexed feature rows: a sparse tensor is
 * an int32 (N, 4) array of coordinate rows (batch, x, y, z) plus an (N, C)
 * feature array, where coordinate row i owns feature row i and batch is the
 * first column (Torch Lattice docs, "Migrating from TorchSparse", section
 * "Sparse tensor expectations").  The library covers the three convolution
 * families of that page's "Convolution mapping" table:
 *   - SubmConv3d       preserves the input support;
 *   - Conv3d, strided  generates a downsampled support;
 *   - ConvTranspose3d  consumes an existing relation back onto a known support;
 * and the hashing, kernel-map construction and coordinate query that feed
 * them, plus pooling over a relation and dense materialization ("What
 * remains familiar": CUDA kernels cover sparse convolution, pooling, hashing,
 * coordinate query and dense materialization).  Forward, data-gradient and per-offset
 * weight-gradient passes are provided, since models train with standard
 * optimizers (same page) and TorchSparse++ targets training as well as
 * inference (TorchSparse++ abstract).
 *
 * Conventions shared by every entry point
 *   - Every pointer is a DEVICE pointer to a caller-allocated, contiguous,
 *     row-major buffer, unless documented as host.  The library never
 *     allocates or frees memory and keeps no state between calls except
 *     per-device kernel attributes set on first use.
 *   - Work is enqueued on `stream` (NULL = legacy default stream) and is
 *     asynchronous, except lat_downsample_coords, lat_upsample_coords and
 *     lat_status_fetch, which synchronise `stream` because they return a
 *     device-computed value.
 *   - Argument errors are detected on the host and returned synchronously;
 *     nothing is enqueued then.  Errors found by a kernel (range, duplicate,
 *     table full, capacity, malformed map) are OR-ed into the caller's int32
 *     status word `d_status` (device memory, may be NULL to ignore) and read
 *     back with lat_status_fetch.
 *   - Scratch memory (`ws`, `ws_bytes`) is supplied by the caller; each op
 *     has a *_ws_bytes query returning the size it needs.  A NULL `ws` with a
 *     zero size is valid when the query returns 0.
 *   - Feature / weight / output arrays share one element type (lat_dtype),
 *     except the weight gradient, which is always fp32.
 *
 * Readings taken where the pages are silent (the same readings drive the
 * CPU oracle used by the tests):
 *   - cross-correlation: y(q) = sum_k x(in(q, k)) * W[k], like dense conv3d;
 *   - offset index k = (ix*Ky + iy)*Kz + iz for offset vector (ix, iy, iz);
 *   - input coordinate of output q at offset k: stride*q + (ix,iy,iz) - pad
 *     (SubmConv3d: stride 1, pad (K-1)/2);
 *   - weights are (K^3, Cin, Cout) row-major; no bias;
 *   - the transposed relation links fine output p to coarse input q when
 *     stride*q + (ix,iy,iz) - pad == p;
 *   - a 16-bit output is the fp32 accumulator rounded to nearest even once.
 */
#ifndef LATTICE_H
#define LATTICE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st *lat_stream;

/* Status codes.  Values are bit flags so a device status word can hold several. */
typedef enum {
    LAT_OK = 0,
    LAT_ERR_ARG = 1,          /* invalid argument (host check)                          */
    LAT_ERR_COORD_RANGE = 2,  /* coordinate outside the packable key range (device)     */
    LAT_ERR_DUPLICATE = 4,    /* two coordinate rows are equal (device)                 */
    LAT_ERR_TABLE_FULL = 8,   /* hash probing visited every slot (device)               */
    LAT_ERR_CAPACITY = 16,    /* an output buffer is smaller than the result (device)   */
    LAT_ERR_UNSUPPORTED = 32, /* shape / dtype combination not implemented (host)       */
    LAT_ERR_CUDA = 64,        /* a CUDA runtime call failed (host)                      */
    LAT_ERR_WORKSPACE = 128,  /* ws_bytes smaller than the *_ws_bytes query (host)      */
    LAT_ERR_BAD_MAP = 256,    /* a kernel map holds a row index outside [0, n_in) (device) */
    LAT_ERR_TIMEOUT = 512     /* a bounded in-kernel wait gave up; the kernel drained and exited */
} lat_status;

typedef enum { LAT_F32 = 0, LAT_F16 = 1, LAT_BF16 = 2 } lat_dtype;

/* Support semantics ("Convolution mapping" table of the migration page). */
typedef enum {
    LAT_SUBM = 0,       /* SubmConv3d: output coords are the input coords themselves  */
    LAT_STRIDED = 1,    /* Conv3d with stride: output coords from lat_downsample_coords */
    LAT_TRANSPOSED = 2  /* ConvTranspose3d: fine outputs, coarse inputs               */
} lat_mode;

/* Convolution geometry.  K^3 = ksize[0]*ksize[1]*ksize[2] must be in [1, 32]. */
typedef struct {
    int32_t ksize[3];
    int32_t stride[3]; /* all 1 for LAT_SUBM                                  */
    int32_t pad[3];    /* LAT_SUBM: (K-1)/2 per axis, K odd                    */
    int32_t mode;      /* lat_mode                                             */
} lat_geom;

/* Rows per output tile of the convolution kernels (and of tile_mask). */
#define LAT_TILE_ROWS 128

/*
 * Kernel map ("relation" in the migration page's "Backend and configuration
 * differences" section): for every output row j and offset k, the input row
 * found at the offset coordinate.  All arrays are caller-allocated device
 * buffers that lat_kmap_query fills:
 *   nbr       int32  [k3][n_out]  nbr[k*n_out + j] = input row, or -1
 *   mask      uint32 [n_out]      bit k set iff nbr[k*n_out + j] >= 0
 *   perm      int32  [n_out]      output rows sorted by the grouping key
 *                                 (min(popcount(mask), 31) << 11) |
 *                                 ((mask * 0x9E3779B1 mod 2^32) >> 21), stable
 *                                 (ties keep ascending row order); rows with
 *                                 equal masks are adjacent.  With k3 <= 8
 *                                 the key is the mask itself.
 *   tile_mask uint32 [ceil(n_out/LAT_TILE_ROWS)]  OR of mask over each run of
 *                                 LAT_TILE_ROWS consecutive entries of perm
 *   pair_off  int64  [k3 + 1]     pair_off[k] = first pair of offset k
 *   pair_in   int32  [pair_capacity]  input row of each pair
 *   pair_out  int32  [pair_capacity]  output row of each pair
 * Pairs are grouped by offset (ascending k) and, within an offset, sorted by
 * ascending output row, so the lists are deterministic.  n_in, n_out and k3
 * are set by the caller before lat_kmap_query; mode records the geometry's
 * mode (written by the query).  In a LAT_SUBM map the centre offset K^3/2
 * maps every row to itself (nbr[centre*n_out + j] == j); the convolution
 * passes rely on that and do not read the centre column.
 */
typedef struct {
    int32_t *nbr;
    uint32_t *mask;
    int32_t *perm;
    uint32_t *tile_mask;
    int64_t *pair_off;
    int32_t *pair_in;
    int32_t *pair_out;
    int64_t pair_capacity;
    int64_t n_in;
    int64_t n_out;
    int32_t k3;
    int32_t mode;
} lat_kmap;

/* ---------------------------------------------------------------- hashing --
 * GPU open-addressing hash of packed 64-bit coordinate keys ("hashing" in
 * the CUDA kernel list of the migration page; capacity knob
 * torch_lattice.backends.hash_rsv_ratio of "Backend and configuration
 * differences").
 *
 * Key packing: key = b<<48 | (x+2^15)<<32 | (y+2^15)<<16 | (z+2^15), so the
 * unsigned key order is the lexicographic (b, x, y, z) order.  b must lie in
 * [0, 65534] and x, y, z in [-32768, 32767]; rows outside are skipped and
 * flag LAT_ERR_COORD_RANGE.  The table holds a power-of-two number of
 * slots, 16 bytes of table each, stored as 64-byte groups of 4 slots
 * {uint64 key[4]; uint32 row[4]; uint32 unused[4]}: slot s is entry s % 4
 * of group s / 4.  An empty slot holds key 0xFFFF...F.  A key's home slot is
 * a 32-bit mix of its z-brick -- the key with the two low bits of the z
 * field cleared, so the 4 cells z = 4m..4m+3 of one (b, x, y) column share
 * it -- (the two halves folded, then the MurmurHash3 fmix32 finalizer)
 * masked to the slot count; its probe sequence starts at the first slot of
 * the home slot's group and runs over consecutive slots (linear probing), so
 * a lookup reads whole groups, and one group read answers the z-neighbours
 * of a cell that share its brick.  A key is stored within
 * 4096 slots of the start of its home group (anywhere in a smaller table);
 * an insert that finds no free slot in that window flags
 * LAT_ERR_TABLE_FULL (only a table filled close to capacity gets there), and
 * a lookup stops after the window.  The table must be 64-byte aligned.
 */

/* Bytes of a table for n rows: 16 * next_pow2(max(ceil(rsv_ratio*n), 64)).
 * rsv_ratio must be >= 1; at most 2^31 slots.  The Python helpers use 4: at
 * a load factor of 1/8..1/4 most probes end at their home slot, which cuts
 * the query's probe rounds.  Returns 0 on invalid input. */
size_t lat_hash_bytes(int64_t n, float rsv_ratio);

/* Insert coords[0..n) (int32 (n,4)) into `table` (table_bytes from
 * lat_hash_bytes; clears it first).  A duplicate coordinate keeps the lowest
 * row and flags LAT_ERR_DUPLICATE; a key with no free slot in its probe
 * window flags LAT_ERR_TABLE_FULL. */
lat_status lat_hash_build(const int32_t *coords, int64_t n, void *table, size_t table_bytes,
                          int32_t *d_status, lat_stream stream);

/* ------------------------------------------------------ kernel-map query --
 * For every output row and each of the K^3 offsets, probe the input table
 * (built by lat_hash_build over the n_in input rows) and fill `map` (see
 * lat_kmap).  Coordinate query + kernel-map construction of the migration
 * page ("What remains familiar"; "Sparse tensor expectations").
 *   LAT_SUBM       out_coords must be the input coordinate rows themselves.
 *   LAT_STRIDED    out_coords come from lat_downsample_coords (same geom).
 *   LAT_TRANSPOSED table holds the coarse rows, out_coords the fine rows.
 * pair_capacity may be as large as n_out*k3; pairs beyond it are dropped and
 * flag LAT_ERR_CAPACITY (pair_off is still exact). */
size_t lat_kmap_ws_bytes(int64_t n_out, int32_t k3);
lat_status lat_kmap_query(const void *table, size_t table_bytes, const int32_t *out_coords,
                          const lat_geom *geom, lat_kmap *map, void *ws, size_t ws_bytes,
                          int32_t *d_status, lat_stream stream);

/* --------------------------------------------------- support generation --
 * Output support of a strided Conv3d ("Convolution mapping": strided forward
 * convolution creates a downsampled support): every coarse q whose window
 * {stride*q + (ix,iy,iz) - pad} holds at least one active input, batch
 * unchanged.  Written to out_coords (int32 (out_capacity, 4)) sorted by packed
 * key, i.e. in canonical (b, x, y, z) order, so the result is deterministic.
 * geom->mode must be LAT_STRIDED.  A bitmap counting sort runs when the
 * coarse fields, shifted to their minimum, pack into at most 30 bits (and the
 * bitmap fits the budget of max(2^24, 512 bits per candidate)); otherwise a
 * radix sort of the packed keys.  Synchronises `stream` once (twice when the
 * radix sort is needed) and writes the row count to *n_out (HOST pointer).
 * out_capacity >= n_in is enough when ksize == stride
 * and pad == 0; in general n_in * prod(ceil(ksize/stride)) bounds the count.
 * Too small a capacity returns LAT_ERR_CAPACITY with the needed count in
 * *n_out.  parent (device int32 [n_in], may be NULL) receives the coarse row
 * of every input row; it needs ksize == stride and pad == 0 (each input then
 * lies in exactly one window), else LAT_ERR_UNSUPPORTED. */
size_t lat_downsample_ws_bytes(int64_t n_in, const lat_geom *geom);
lat_status lat_downsample_coords(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                                 int32_t *out_coords, int64_t out_capacity, int64_t *n_out,
                                 int32_t *parent, void *ws, size_t ws_bytes, int32_t *d_status,
                                 lat_stream stream);

/* The same support without waiting: enqueues the bitmap counting sort and a
 * copy of the row count into *n_out_host, then returns.  n_out_host should be
 * pinned host memory (cudaHostAlloc), else the copy may synchronise.  Once
 * `stream` has passed this point (an event recorded after the call), *n_out_host
 * holds the row count, or -1 when the coarse fields do not fit the bitmap:
 * then call lat_downsample_coords with the same arguments.  Rows beyond
 * out_capacity are not written; a count above out_capacity means the buffer
 * was too small.  out_coords, parent and ws must stay untouched until then. */
lat_status lat_downsample_coords_async(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                                       int32_t *out_coords, int64_t out_capacity, int64_t *n_out_host,
                                       int32_t *parent, void *ws, size_t ws_bytes, int32_t *d_status,
                                       lat_stream stream);

/* Output support of a GenerativeConvTranspose3d (migration page, "Convolution
 * mapping": a generative transposed convolution creates its output support):
 * every fine coordinate s*q + (ix,iy,iz) - pad for an input (coarse) row q and
 * offset (ix,iy,iz) in [0,K)^3, batch unchanged, made unique and written to
 * out_coords in canonical (b, x, y, z) order.  geom->mode must be
 * LAT_TRANSPOSED (the geometry the transposed map of the same conv uses).
 * Generated coordinates outside the packable key range are dropped and flag
 * LAT_ERR_COORD_RANGE.  out_capacity >= n_in * K^3 always suffices.  Same
 * algorithm, synchronisation and errors as lat_downsample_coords (no parents).
 * The convolution then runs on lat_kmap_query(table of the input rows,
 * out_coords, LAT_TRANSPOSED geom). */
size_t lat_upsample_ws_bytes(int64_t n_in, const lat_geom *geom);
lat_status lat_upsample_coords(const int32_t *coords, int64_t n_in, const lat_geom *geom,
                               int32_t *out_coords, int64_t out_capacity, int64_t *n_out, void *ws,
                               size_t ws_bytes, int32_t *d_status, lat_stream stream);

/* Both kernel maps of a strided Conv3d with ksize == stride and pad == 0,
 * built from the parent rows that lat_downsample_coords reports instead of by
 * probing: fine row i sits in coarse window parent[i] at offset
 * k(i) = (o0*Ky + o1)*Kz + o2 with o = fine coordinate mod stride (floor).
 *   down  LAT_STRIDED map: n_out = coarse rows, n_in = fine rows
 *         (nbr[k(i)][parent[i]] = i);
 *   up    LAT_TRANSPOSED map: n_out = fine rows, n_in = coarse rows
 *         (nbr[k][i] = parent[i] if k == k(i), else -1).
 * Either map may be NULL.  The caller sets n_in / n_out / k3 of each map; the
 * results equal what lat_kmap_query returns for the same geometry. */
size_t lat_kmap_from_parent_ws_bytes(int64_t n_fine, int64_t n_coarse, int32_t k3);
lat_status lat_kmap_from_parent(const int32_t *fine_coords, const int32_t *parent, const lat_geom *geom,
                                lat_kmap *down, lat_kmap *up, void *ws, size_t ws_bytes,
                                int32_t *d_status, lat_stream stream);

/* ------------------------------------------------------------ convolution --
 * y[j] = sum over k with nbr[k][j] >= 0 of x[nbr[k][j]] . W[k]
 * x (map->n_in, cin), w (k3, cin, cout), y (map->n_out, cout), all `dtype`;
 * accumulation in fp32; every output row is written exactly once (rows with
 * no neighbour get zeros).  Implicit-GEMM dataflow (TorchSparse++ abstract;
 * the migration page requires every dataflow to give the same result for a
 * fixed relation and weight tensor).  cin and cout must be multiples of 8 and
 * at most 256.  fp16 / bf16 with cin, cout in {64, 128} run on the tcgen05
 * tensor cores (fp32 accumulate in TMEM); other shapes and fp32 run on CUDA
 * cores (FFMA, no TF32).
 * Workspace: the tensor-core forward and data-gradient passes take 256 bytes
 * (a tile counter, cleared on `stream` before the kernel); the CUDA-core
 * passes take none.  lat_sconv_ws_bytes gives the size for each op; a call
 * with less returns LAT_ERR_WORKSPACE.  Two calls must not share a workspace
 * while both can run (different streams). */
size_t lat_sconv_ws_bytes(int32_t op, int32_t cin, int32_t cout, const lat_kmap *map,
                          lat_dtype dtype);
#define LAT_OP_FWD 0
#define LAT_OP_DGRAD 1
#define LAT_OP_WGRAD 2
lat_status lat_sconv_fwd(const void *x, int32_t cin, const void *w, int32_t cout,
                         const lat_kmap *map, void *y, lat_dtype dtype, void *ws, size_t ws_bytes,
                         int32_t *d_status, lat_stream stream);

/* Data gradient: dx[i] = sum over pairs (i, j, k) of dy[j] . W[k]^T.
 * `map` is the relation seen from dx's rows:
 *   SubmConv3d        pass the forward map and flip_offsets = 1 (the pair
 *                     (i, j, k) is found at nbr[k3-1-k][i]);
 *   strided Conv3d    pass the LAT_TRANSPOSED map of the same geometry
 *                     (fine rows as outputs), flip_offsets = 0;
 *   ConvTranspose3d   pass the LAT_STRIDED map, flip_offsets = 0.
 * dy (map->n_in... rows of the forward output, cout), w (k3, cin, cout) as in
 * the forward pass, dx (map->n_out, cin). */
lat_status lat_sconv_dgrad(const void *dy, int32_t cout, const void *w, int32_t cin,
                           const lat_kmap *map, int32_t flip_offsets, void *dx, lat_dtype dtype,
                           void *ws, size_t ws_bytes, int32_t *d_status, lat_stream stream);

/* Per-offset weight gradient: dW[k] = sum over pairs (i, j) of offset k of
 * x[i]^T dy[j], fp32 (k3, cin, cout), from the forward map's pair lists.
 * Deterministic: the pair list is cut into a fixed number of equal
 * contiguous shares (296 on the tensor cores; on the CUDA cores 1184 when
 * cin*cout <= 2048, else 296; never more shares than pairs), each share is
 * reduced into fp32 partials (one per offset it meets), and the partials are
 * summed in a fixed order (no atomics), so the bits do not depend on timing,
 * on the number of SMs or on pair_capacity.  The scratch holds
 * (shares + k3) partials of cin*cout fp32, whatever the pair count. */
lat_status lat_sconv_wgrad(const void *x, int32_t cin, const void *dy, int32_t cout,
                           const lat_kmap *map, float *dw, lat_dtype dtype, void *ws,
                           size_t ws_bytes, int32_t *d_status, lat_stream stream);

/* Weight gradient for callers that cannot allocate.  No counterpart in the
 * papers or docs: this exists for users of the library, not for the method.
 *
 * Some callers cannot call cudaMalloc or hand over a scratch buffer: code
 * that runs while a stream is captured into a CUDA graph without memory
 * nodes, real-time loops that must not allocate (cudaMalloc / cudaFree can
 * synchronise the whole device) once running, or hosts whose device
 * allocator belongs to another runtime.  This entry point computes dW with
 * the CUDA-core weight-gradient kernels (those lat_sconv_wgrad runs for fp32
 * and for the shapes the tensor cores do not take; same shares, same
 * summation order, so the same bits there; for the tensor-core shapes of
 * lat_sconv_wgrad the two agree within fp32 rounding, not bit for bit) and
 * takes no `ws`: its scratch is one static device array of
 * LAT_WGRAD_STATIC_SCRATCH_BYTES (32 MiB) inside the library, which every
 * GPU that loads the library keeps until the process exits.  It allocates
 * nothing and calls no allocating routine.
 *   - Limit: the scratch must hold (shares + k3) fp32 partials of cin*cout
 *     (shares as for lat_sconv_wgrad above); it does not depend on the row
 *     or pair count.  With k3 = 27 that allows cin*cout up to 25,970 (every
 *     shape up to 128 x 192); larger shapes return LAT_ERR_WORKSPACE before
 *     anything is enqueued.
 *   - The first successful call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and keeps it;
 *     make that first call before any stream capture begins.  A failed
 *     lookup returns LAT_ERR_CUDA and is tried again on the next call.
 *   - All calls share the one array and it keeps the last call's contents;
 *     every byte a call reads is written earlier by the same call, so no
 *     clearing is needed.  Calls whose work overlaps on the GPU (different
 *     streams, or host threads racing on one device) race on the array:
 *     order them on one stream. */
#define LAT_WGRAD_STATIC_SCRATCH_BYTES (32u << 20)
lat_status lat_sconv_wgrad_static(const void *x, int32_t cin, const void *dy, int32_t cout,
                                  const lat_kmap *map, float *dw, lat_dtype dtype,
                                  int32_t *d_status, lat_stream stream);

/* ------------------------------------------- pooling and dense grids --- */

typedef enum { LAT_POOL_MAX = 0, LAT_POOL_AVG = 1 } lat_pool_op;

/* Sparse pooling over a kernel map ("What remains familiar" of the
 * migration page: pooling is one of the library's CUDA kernels; the pages
 * give no formula, so the plain reading is taken).  For every output row j:
 *   y[j][c] = max  over { x[nbr[k*n_out + j]][c] : bit k of mask[j] set }
 *   y[j][c] = mean over the same set (fp32 sum in ascending k, divided by
 *             the number of neighbours)
 * and y[j] = 0 where mask[j] == 0.  The map is any map lat_kmap_query or
 * lat_kmap_from_parent built (SUBM, strided or transposed geometry); only
 * nbr and mask are read, with map->n_in / n_out / k3 giving the sizes.
 *   x  device [n_in][c] of dtype; y device [n_out][c] of dtype (no overlap
 *      with x).  Both 16-byte aligned; c a multiple of 8 in [8, 2048].
 *   Arithmetic is fp32; each output is rounded once to dtype.
 *   op is lat_pool_op.  Host checks return LAT_ERR_ARG; a row index outside
 *   [0, n_in) or a mask bit at or above k3 sets LAT_ERR_BAD_MAP at d_status
 *   (may be NULL) and that neighbour is skipped.  Asynchronous on `stream`; allocates nothing. */
lat_status lat_sparse_pool(const void *x, int32_t c, const lat_kmap *map, int32_t op, void *y,
                           lat_dtype dtype, int32_t *d_status, lat_stream stream);

/* Dense materialization (same passage): write the sparse tensor into a
 * zero-filled channels-last grid out[batch][shape[0]][shape[1]][shape[2]][c]
 * of dtype covering x in [origin[0], origin[0]+shape[0]) and likewise for
 * y and z, batches 0..batch-1.  Row i lands in cell
 * (b, x-origin[0], y-origin[1], z-origin[2]) of coords[i] = (b,x,y,z); a row
 * outside the box is skipped and sets LAT_ERR_COORD_RANGE at d_status.
 * Coordinates are expected unique (as after hashing); with duplicates one
 * of the rows wins, which one is unspecified.
 *   coords device int32 [n][4], 16-byte aligned; feats device [n][c];
 *   origin, shape host int32[3]; out device, 16-byte aligned,
 *   batch*shape[0]*shape[1]*shape[2]*c elements.  c a multiple of 8 in
 *   [8, 2048]; n < 2^31.
 * Enqueues a memset of `out` and one scatter kernel on `stream`. */
lat_status lat_to_dense(const int32_t *coords, int64_t n, const void *feats, int32_t c, lat_dtype dtype,
                        const int32_t *origin, const int32_t *shape, int32_t batch, void *out,
                        int32_t *d_status, lat_stream stream);

/* ---------------------------------------------------------------- misc --- */

/* Synchronise `stream`, then return the status word at d_status (device). */
int32_t lat_status_fetch(const int32_t *d_status, lat_stream stream);

/* Static description of a status value (bit flags are listed by lowest bit). */
const char *lat_status_string(int32_t status);

/* Library ABI version (major*100 + minor). */
int32_t lat_version(void);

/* Failure detection: limit, in nanoseconds, of every barrier wait in the
 * tensor-core kernels (the fp16 / bf16 convolution and weight-gradient
 * passes); 2 s by default.  A wait that runs out flags LAT_ERR_TIMEOUT at
 * d_status; its CTA then waits (with a separate 1 s limit) for the tensor
 * memory accelerator loads and MMAs it still has in flight, frees its tensor
 * memory and exits, so the context stays usable and later calls run
 * normally.  The outputs of a call that timed out are undefined.  0 makes
 * every wait that is not already complete give up at once (tests use it to
 * run the timeout path without faulting or hanging anything).  One
 * process-wide value, read at each launch; returns the previous one. */
uint64_t lat_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* LATTICE_H */
