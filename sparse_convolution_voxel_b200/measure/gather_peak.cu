// Random-row copy throughput of the device (a measurement kernel, not part
// of the convolution library).
//
// The convolution passes read their operand rows in the order of a kernel
// map and write their output rows in the order of the mask-sorted tiles:
// both are rows of a few hundred bytes at scattered addresses, a pattern that
// the STREAM-style copy of the measured HBM peak does not exercise.  This
// kernel copies rows dst[out_idx[i]] = src[in_idx[i]] (out_idx NULL: row i),
// 16 bytes per thread per step, consecutive threads on consecutive chunks of
// a row, grid-stride over the rows, so its throughput is the memory system's
// rate for that pattern alone.  Bytes per launch = 2 * n * row_bytes plus the
// index words.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lattice_measure.h"

namespace {

__global__ void __launch_bounds__(256) gather_kernel(const uint4 *__restrict__ src, const int32_t *__restrict__ in_idx,
                                                     const int32_t *__restrict__ out_idx, int64_t n, int chunks,
                                                     uint4 *__restrict__ dst) {
    const int64_t total = n * chunks;
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
         e += int64_t(gridDim.x) * blockDim.x) {
        const int64_t i = e / chunks;
        const int c = int(e - i * chunks);
        const int64_t r = __ldg(in_idx + i);
        const int64_t o = out_idx ? int64_t(__ldg(out_idx + i)) : i;
        dst[o * chunks + c] = __ldg(src + r * chunks + c);
    }
}

}  // namespace

extern "C" int lat_measure_gather(const void *src, const int32_t *in_idx, const int32_t *out_idx, int64_t n,
                                  int row_bytes, void *dst, int blocks, void *stream) {
    if (!src || !in_idx || !dst || n < 0 || row_bytes < 16 || row_bytes % 16 || blocks < 1) return 1;
    if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 16) return 1;
    if (n == 0) return 0;
    gather_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(src), in_idx, out_idx, n, row_bytes / 16, static_cast<uint4 *>(dst));
    return cudaGetLastError() == cudaSuccess ? 0 : 64;
}
