/*
 * lattice_measure.h -- measurement kernels shipped beside liblattice.so
 * (libmeasure.so).  They are not part of the convolution path: the benchmark
 * uses them to measure device rates that the rooflines need and that no
 * library routine provides (the fp32 FMA rate of the CUDA-core path, the
 * random-row copy rate of the gathered operands).
 */
#ifndef LATTICE_MEASURE_H
#define LATTICE_MEASURE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* FP32 FMA throughput probe: launches `blocks` x `threads` threads (threads a
 * multiple of 32, at most 256) on `stream` (a cudaStream_t, NULL = default),
 * each running `iters` loop trips of independent fmaf(v, m, c) chains, and
 * stores one float per thread into `out` (device, blocks*threads floats).
 * Returns 0, 1 for a bad argument, 64 for a launch error.  The caller times
 * the launch; lat_measure_ffma_flops gives the FLOPs it performs. */
int lat_measure_ffma(float *out, int blocks, int threads, int iters, float m, float c, void *stream);

/* FLOPs (2 per FMA) of one lat_measure_ffma launch with these sizes. */
double lat_measure_ffma_flops(int blocks, int threads, int iters);

/* Random-row copy probe: dst[out_idx[i]] = src[in_idx[i]] for i < n, rows of
 * row_bytes bytes (a multiple of 16; src and dst 16-byte aligned device
 * buffers, in_idx / out_idx device int32 arrays of n valid row indices;
 * out_idx NULL writes row i).  `blocks` blocks of 256 threads, grid-stride,
 * on `stream`.  Returns 0, 1 for a bad argument, 64 for a launch error.  It
 * reads and writes 2 * n * row_bytes bytes of rows plus the index words; the
 * caller times it. */
int lat_measure_gather(const void *src, const int32_t *in_idx, const int32_t *out_idx, int64_t n, int row_bytes,
                       void *dst, int blocks, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LATTICE_MEASURE_H */
