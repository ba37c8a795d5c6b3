// FP32 fused multiply-add throughput of the device (a measurement kernel, not
// part of the convolution library).
//
// The fp32 convolutions run on the CUDA cores, so their roofline needs the
// device's FFMA rate as well as its memory bandwidth.  Every thread runs
// kChains independent chains of fmaf(v, m, c), kUnroll steps per loop trip,
// so each warp scheduler always has independent FMAs to issue; the operands m
// and c are kernel arguments, so nothing can be folded at compile time, and
// every thread stores its sum, so no chain is dead code.  FLOPs per launch =
// 2 * kChains * kUnroll * iters * threads.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lattice_measure.h"

namespace {

constexpr int kChains = 8;
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(256) ffma_kernel(float *__restrict__ out, int iters, float m, float c) {
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    float v[kChains];
#pragma unroll
    for (int j = 0; j < kChains; ++j) v[j] = 1e-3f * float(threadIdx.x + j);
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
            for (int j = 0; j < kChains; ++j) v[j] = fmaf(v[j], m, c);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kChains; ++j) s += v[j];
    out[tid] = s;
}

}  // namespace

extern "C" int lat_measure_ffma(float *out, int blocks, int threads, int iters, float m, float c, void *stream) {
    if (!out || blocks < 1 || threads < 32 || threads > 256 || threads % 32 || iters < 1) return 1;
    ffma_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(out, iters, m, c);
    return cudaGetLastError() == cudaSuccess ? 0 : 64;
}

extern "C" double lat_measure_ffma_flops(int blocks, int threads, int iters) {
    return 2.0 * kChains * kUnroll * double(iters) * double(blocks) * double(threads);
}
