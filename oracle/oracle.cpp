// Plain CPU oracle for sparse convolution over coordinate-indexed voxels.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load this
// library: only the tests, the package's smoke check and the CPU-baseline
// leg of the benchmark do.  It shares no code, header, table or constant
// with the CUDA library; both sides read the same seeded inputs.
//
// What it computes, and where that is defined:
//   * A sparse tensor is a set of integer rows (batch, x, y, z) with one
//     feature row per coordinate row; batch is the first column and is never
//     changed by a convolution ("Migrating from TorchSparse", section
//     "Sparse tensor expectations").
//   * The kernel map ("relation") lists, for each output row and each kernel
//     offset, the input row found at the offset coordinate ("Migrating from
//     TorchSparse", sections "Convolution mapping" and "Backend and
//     configuration differences": hashing, kernel-map construction and
//     coordinate query).  It is built here with a std::unordered_map.
//   * SubmConv3d keeps the input support; strided Conv3d generates a
//     coarser support; ConvTranspose3d consumes an existing relation
//     ("Convolution mapping" table).
//   * The convolution result is the plain gather-scatter sum over the
//     relation, accumulated in fp64.  The docs page states that implicit
//     GEMM, fetch-on-demand and gather-scatter compute the same sparse result
//     for a fixed relation and weight tensor ("Backend and configuration
//     differences"); TorchSparse++'s abstract names gather-GEMM-scatter as the
//     simple dataflow.  So the plain sum is the definition the fast path must
//     reproduce up to rounding order.
//   * Pooling and dense materialization are listed among the library's
//     kernels ("What remains familiar") with no formula: pooling here is the
//     max or mean over the same relation, dense materialization the scatter
//     of each row into a zeroed grid.
//
// Readings where the pages are silent (each is listed in the design notes):
//   * cross-correlation: y(q) = sum_k x(in(q,k)) * W[k], as dense conv3d;
//   * offset order k = (ix*Ky + iy)*Kz + iz, offset vector (ix,iy,iz);
//   * input coordinate of (output q, offset k): s*q + (ix,iy,iz) - pad
//     (submanifold: s = 1, pad = (K-1)/2);
//   * transposed relation: output p (fine), input q (coarse), linked when
//     s*q + (ix,iy,iz) - pad == p;
//   * packed key (b<<48)|(x+2^15)<<32|(y+2^15)<<16|(z+2^15), so unsigned key
//     order equals lexicographic (b,x,y,z) order; b must lie in [0, 65534],
//     x,y,z in [-32768, 32767].
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <cmath>
#include <set>
#include <unordered_map>
#include <vector>
#include <omp.h>

namespace {

constexpr int ORC_OK = 0;
constexpr int ORC_RANGE = 2;
constexpr int ORC_DUPLICATE = 3;
constexpr int ORC_ARG = 1;

enum Mode { SUBM = 0, STRIDED = 1, TRANSPOSED = 2 };

bool in_range(int64_t b, int64_t x, int64_t y, int64_t z) {
    return b >= 0 && b <= 65534 && x >= -32768 && x <= 32767 && y >= -32768 && y <= 32767 &&
           z >= -32768 && z <= 32767;
}

uint64_t pack(int64_t b, int64_t x, int64_t y, int64_t z) {
    return (uint64_t(b) << 48) | (uint64_t(x + 32768) << 32) | (uint64_t(y + 32768) << 16) |
           uint64_t(z + 32768);
}

void unpack(uint64_t key, int32_t* c) {
    c[0] = int32_t(key >> 48);
    c[1] = int32_t((key >> 32) & 0xFFFF) - 32768;
    c[2] = int32_t((key >> 16) & 0xFFFF) - 32768;
    c[3] = int32_t(key & 0xFFFF) - 32768;
}

// floor division / floor modulo for possibly negative numerators
int64_t fdiv(int64_t a, int64_t b) { int64_t q = a / b; if ((a % b != 0) && ((a < 0) != (b < 0))) --q; return q; }
int64_t fmod_(int64_t a, int64_t b) { return a - fdiv(a, b) * b; }

void set_threads(int nthreads) {
    if (nthreads > 0) omp_set_num_threads(nthreads);
}

}  // namespace

extern "C" {

int orc_version() { return 1; }

// Packed key of one coordinate row; returns ~0 if out of range.
uint64_t orc_pack_key(int32_t b, int32_t x, int32_t y, int32_t z) {
    if (!in_range(b, x, y, z)) return ~uint64_t(0);
    return pack(b, x, y, z);
}

// Kernel map.  nbr is [n_out][k3] row-major: nbr[j*k3 + k] = input row or -1.
// Returns ORC_OK, ORC_RANGE (an input coordinate outside the key range),
// ORC_DUPLICATE (two input rows with the same coordinate) or ORC_ARG.
int orc_kmap(const int32_t* in_coords, int64_t n_in, const int32_t* out_coords, int64_t n_out,
             const int32_t* ksize, const int32_t* stride, const int32_t* pad, int mode,
             int32_t* nbr, int nthreads) {
    if (mode < SUBM || mode > TRANSPOSED) return ORC_ARG;
    for (int a = 0; a < 3; ++a)
        if (ksize[a] < 1 || stride[a] < 1) return ORC_ARG;
    const int k3 = ksize[0] * ksize[1] * ksize[2];
    std::unordered_map<uint64_t, int32_t> table;
    table.reserve(size_t(n_in) * 2);
    for (int64_t i = 0; i < n_in; ++i) {
        const int32_t* c = in_coords + 4 * i;
        if (!in_range(c[0], c[1], c[2], c[3])) return ORC_RANGE;
        if (!table.emplace(pack(c[0], c[1], c[2], c[3]), int32_t(i)).second) return ORC_DUPLICATE;
    }
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n_out; ++j) {
        const int32_t* q = out_coords + 4 * j;
        for (int ix = 0; ix < ksize[0]; ++ix)
            for (int iy = 0; iy < ksize[1]; ++iy)
                for (int iz = 0; iz < ksize[2]; ++iz) {
                    const int k = (ix * ksize[1] + iy) * ksize[2] + iz;
                    const int off[3] = {ix, iy, iz};
                    int64_t p[3];
                    bool ok = true;
                    for (int a = 0; a < 3; ++a) {
                        const int64_t qa = q[a + 1];
                        if (mode == SUBM) {
                            p[a] = qa + off[a] - pad[a];
                        } else if (mode == STRIDED) {
                            p[a] = int64_t(stride[a]) * qa + off[a] - pad[a];
                        } else {  // TRANSPOSED: find coarse q' with s*q' + off - pad == q
                            const int64_t t = qa - off[a] + pad[a];
                            if (fmod_(t, stride[a]) != 0) ok = false;
                            p[a] = fdiv(t, stride[a]);
                        }
                    }
                    int32_t found = -1;
                    if (ok && in_range(q[0], p[0], p[1], p[2])) {
                        auto it = table.find(pack(q[0], p[0], p[1], p[2]));
                        if (it != table.end()) found = it->second;
                    }
                    nbr[j * k3 + k] = found;
                }
    }
    return ORC_OK;
}

// Support generated by a strided convolution: every coarse q whose window
// {s*q + off - pad : off in [0,K)^3} holds at least one active input.
// Writes the coarse rows sorted by packed key (canonical order) into out
// (capacity rows) and returns their count, or -1 on a bad argument / range
// error, or -(needed) - 2 if capacity is too small.
int64_t orc_downsample(const int32_t* coords, int64_t n, const int32_t* ksize,
                       const int32_t* stride, const int32_t* pad, int32_t* out, int64_t capacity) {
    for (int a = 0; a < 3; ++a)
        if (ksize[a] < 1 || stride[a] < 1) return -1;
    std::set<uint64_t> support;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t* c = coords + 4 * i;
        if (!in_range(c[0], c[1], c[2], c[3])) return -1;
        for (int ix = 0; ix < ksize[0]; ++ix)
            for (int iy = 0; iy < ksize[1]; ++iy)
                for (int iz = 0; iz < ksize[2]; ++iz) {
                    const int off[3] = {ix, iy, iz};
                    int64_t q[3];
                    bool ok = true;
                    for (int a = 0; a < 3; ++a) {
                        const int64_t t = int64_t(c[a + 1]) - off[a] + pad[a];
                        if (fmod_(t, stride[a]) != 0) ok = false;
                        q[a] = fdiv(t, stride[a]);
                    }
                    if (ok && in_range(c[0], q[0], q[1], q[2])) support.insert(pack(c[0], q[0], q[1], q[2]));
                }
    }
    const int64_t m = int64_t(support.size());
    if (m > capacity) return -m - 2;
    int64_t r = 0;
    for (uint64_t key : support) unpack(key, out + 4 * r++);
    return m;
}

// Support generated by a transposed convolution: every s*q + off - pad for an
// input (coarse) row q and off in [0,K)^3, batch unchanged, in range only,
// sorted by packed key (migration page, "Convolution mapping": generative
// transposed convolutions create their output support).
int64_t orc_upsample(const int32_t* coords, int64_t n, const int32_t* ksize,
                     const int32_t* stride, const int32_t* pad, int32_t* out, int64_t capacity) {
    for (int a = 0; a < 3; ++a)
        if (ksize[a] < 1 || stride[a] < 1) return -1;
    std::set<uint64_t> support;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t* c = coords + 4 * i;
        if (!in_range(c[0], c[1], c[2], c[3])) return -1;
        for (int ix = 0; ix < ksize[0]; ++ix)
            for (int iy = 0; iy < ksize[1]; ++iy)
                for (int iz = 0; iz < ksize[2]; ++iz) {
                    const int off[3] = {ix, iy, iz};
                    int64_t p[3];
                    for (int a = 0; a < 3; ++a) p[a] = int64_t(stride[a]) * c[a + 1] + off[a] - pad[a];
                    if (in_range(c[0], p[0], p[1], p[2])) support.insert(pack(c[0], p[0], p[1], p[2]));
                }
    }
    const int64_t m = int64_t(support.size());
    if (m > capacity) return -m - 2;
    int64_t r = 0;
    for (uint64_t key : support) unpack(key, out + 4 * r++);
    return m;
}

// y[j] = sum over k ascending with i = nbr[j][k] >= 0 of x[i] . W[k]
// x: [n_in][cin], w: [k3][cin][cout], y: [n_out][cout]; all fp64.
void orc_conv_fwd(const double* x, int64_t n_in, int cin, const double* w, int cout,
                  const int32_t* nbr, int64_t n_out, int k3, double* y, int nthreads) {
    (void)n_in;
    set_threads(nthreads);
#pragma omp parallel
    {
        std::vector<double> acc(cout);
#pragma omp for schedule(static)
        for (int64_t j = 0; j < n_out; ++j) {
            std::fill(acc.begin(), acc.end(), 0.0);
            for (int k = 0; k < k3; ++k) {
                const int32_t i = nbr[j * k3 + k];
                if (i < 0) continue;
                const double* xi = x + int64_t(i) * cin;
                const double* wk = w + int64_t(k) * cin * cout;
                for (int ci = 0; ci < cin; ++ci) {
                    const double xv = xi[ci];
                    const double* wr = wk + int64_t(ci) * cout;
                    for (int co = 0; co < cout; ++co) acc[co] += xv * wr[co];
                }
            }
            std::memcpy(y + j * cout, acc.data(), sizeof(double) * cout);
        }
    }
}

// dx[i] = sum over pairs (i, j, k) of dy[j] . W[k]^T  (the adjoint of fwd)
// dy: [n_out][cout], dx: [n_in][cin].  The pairs of each input row are
// visited in ascending (j, k) order.
void orc_conv_dgrad(const double* dy, int64_t n_out, int cout, const double* w, int cin,
                    const int32_t* nbr, int k3, double* dx, int64_t n_in, int nthreads) {
    // inverse relation: for each input row, its (j, k) pairs
    std::vector<int64_t> start(n_in + 1, 0);
    for (int64_t j = 0; j < n_out; ++j)
        for (int k = 0; k < k3; ++k) {
            const int32_t i = nbr[j * k3 + k];
            if (i >= 0) ++start[i + 1];
        }
    for (int64_t i = 0; i < n_in; ++i) start[i + 1] += start[i];
    std::vector<int64_t> fill(start.begin(), start.end() - 1);
    std::vector<int64_t> pj(start[n_in]);
    std::vector<int32_t> pk(start[n_in]);
    for (int64_t j = 0; j < n_out; ++j)
        for (int k = 0; k < k3; ++k) {
            const int32_t i = nbr[j * k3 + k];
            if (i >= 0) { pj[fill[i]] = j; pk[fill[i]] = k; ++fill[i]; }
        }
    set_threads(nthreads);
#pragma omp parallel
    {
        std::vector<double> acc(cin);
#pragma omp for schedule(static)
        for (int64_t i = 0; i < n_in; ++i) {
            std::fill(acc.begin(), acc.end(), 0.0);
            for (int64_t e = start[i]; e < start[i + 1]; ++e) {
                const double* g = dy + pj[e] * cout;
                const double* wk = w + int64_t(pk[e]) * cin * cout;
                for (int ci = 0; ci < cin; ++ci) {
                    const double* wr = wk + int64_t(ci) * cout;
                    double s = 0.0;
                    for (int co = 0; co < cout; ++co) s += g[co] * wr[co];
                    acc[ci] += s;
                }
            }
            std::memcpy(dx + i * cin, acc.data(), sizeof(double) * cin);
        }
    }
}

// dW[k] = sum over pairs (i, j) of offset k of x[i]^T dy[j]   (cin x cout)
// Pairs of each offset are visited in ascending output row j.
void orc_conv_wgrad(const double* x, int cin, const double* dy, int cout, const int32_t* nbr,
                    int64_t n_out, int k3, double* dw, int nthreads) {
    std::memset(dw, 0, sizeof(double) * size_t(k3) * cin * cout);
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t kc = 0; kc < int64_t(k3) * cin; ++kc) {
        const int k = int(kc / cin), ci = int(kc % cin);
        double* row = dw + (int64_t(k) * cin + ci) * cout;
        for (int64_t j = 0; j < n_out; ++j) {
            const int32_t i = nbr[j * k3 + k];
            if (i < 0) continue;
            const double xv = x[int64_t(i) * cin + ci];
            const double* g = dy + j * cout;
            for (int co = 0; co < cout; ++co) row[co] += xv * g[co];
        }
    }
}

// Sparse pooling over a relation (migration page, "What remains familiar":
// pooling is one of the library's kernels; no formula is given, so the plain
// reading): y[j][c] = max, or mean, of x[i][c] over the rows i = nbr[j][k] >= 0,
// k ascending; 0 for a row with no neighbour.  op 0 = max, 1 = mean.  fp64.
void orc_pool(const double* x, int64_t n_in, int c, const int32_t* nbr, int64_t n_out, int k3,
              int op, double* y) {
    (void)n_in;
    for (int64_t j = 0; j < n_out; ++j) {
        double* yj = y + j * c;
        int count = 0;
        for (int k = 0; k < k3; ++k) {
            const int32_t i = nbr[j * k3 + k];
            if (i < 0) continue;
            const double* xi = x + int64_t(i) * c;
            for (int ch = 0; ch < c; ++ch) {
                if (count == 0) yj[ch] = xi[ch];
                else if (op == 0) yj[ch] = std::max(yj[ch], xi[ch]);
                else yj[ch] += xi[ch];
            }
            ++count;
        }
        for (int ch = 0; ch < c; ++ch) {
            if (count == 0) yj[ch] = 0.0;
            else if (op == 1) yj[ch] /= count;
        }
    }
}

// Dense materialization (same passage): out[b][x-ox][y-oy][z-oz][ch] =
// feats[i][ch] for every row i = (b,x,y,z) inside the box, 0 elsewhere.
// Returns the number of rows that fall outside the box (they are skipped).
int64_t orc_to_dense(const int32_t* coords, int64_t n, const double* feats, int c, const int32_t* origin,
                     const int32_t* shape, int batch, double* out) {
    const int64_t cells = int64_t(batch) * shape[0] * shape[1] * shape[2];
    std::memset(out, 0, sizeof(double) * size_t(cells) * c);
    int64_t outside = 0;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t* q = coords + 4 * i;
        int64_t rel[3];
        bool inside = q[0] >= 0 && q[0] < batch;
        for (int a = 0; a < 3; ++a) {
            rel[a] = int64_t(q[a + 1]) - origin[a];
            inside = inside && rel[a] >= 0 && rel[a] < shape[a];
        }
        if (!inside) { ++outside; continue; }
        const int64_t cell = ((int64_t(q[0]) * shape[0] + rel[0]) * shape[1] + rel[1]) * shape[2] + rel[2];
        std::memcpy(out + cell * c, feats + i * c, sizeof(double) * c);
    }
    return outside;
}

int orc_max_threads() { return omp_get_max_threads(); }

}  // extern "C"
