/*
 * lattice_measure.h -- measurement kernels shipped beside liblattice.so
 * (libmeasure.so).  They are not part of the convolution path: the benchmark
 * uses them to measure device peaks that the roofline of the fp32 path needs
 * and that no library routine provides.
 */
#ifndef LATTICE_MEASURE_H
#define LATTICE_MEASURE_H

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

#ifdef __cplusplus
}
#endif

#endif /* LATTICE_MEASURE_H */
