// Device helpers shared by the liblattice kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "lattice.h"

namespace lat {

constexpr uint64_t kEmptyKey = ~0ull;

// The table is an array of 64-byte groups of 4 slots, keys first: one probe
// round reads a group's 4 keys with two 16-byte loads, and the row of a
// matching slot with one more load.  Slot s is entry s % 4 of group s / 4;
// the table size is counted in slots (16 bytes of table each).
constexpr int kGroupSlots = 4;
constexpr size_t kSlotBytes = 16;
struct __align__(64) SlotGroup {
    unsigned long long key[kGroupSlots];
    unsigned int row[kGroupSlots];  // unsigned so atomicMin keeps the lowest row; 0xFFFFFFFF = none
    unsigned int unused[kGroupSlots];
};
static_assert(sizeof(SlotGroup) == kGroupSlots * kSlotBytes, "slot group layout");

// Packed key of (b, x, y, z); returns false when a field is outside the key range.
__device__ __forceinline__ bool pack_key(int b, int x, int y, int z, uint64_t &key) {
    if (b < 0 || b > 65534 || x < -32768 || x > 32767 || y < -32768 || y > 32767 || z < -32768 ||
        z > 32767)
        return false;
    key = (uint64_t(b) << 48) | (uint64_t(x + 32768) << 32) | (uint64_t(y + 32768) << 16) |
          uint64_t(z + 32768);
    return true;
}

__device__ __forceinline__ void unpack_key(uint64_t key, int4 &c) {
    c.x = int(key >> 48);
    c.y = int((key >> 32) & 0xFFFF) - 32768;
    c.z = int((key >> 16) & 0xFFFF) - 32768;
    c.w = int(key & 0xFFFF) - 32768;
}

// Slot hash of a packed key: fold the two 32-bit halves (the high half scaled by
// the 32-bit golden-ratio constant), then the MurmurHash3 32-bit finalizer
// (Austin Appleby, public domain) for full avalanche, so neighbouring voxels land
// in unrelated slots.  32-bit arithmetic only: the probe kernels are
// instruction-bound and slot counts are below 2^31.
__device__ __forceinline__ uint32_t slot_hash(uint64_t key) {
    uint32_t h = uint32_t(key) ^ (uint32_t(key >> 32) * 0x9E3779B1u);
    h ^= h >> 16;
    h *= 0x85EBCA6Bu;
    h ^= h >> 13;
    h *= 0xC2B2AE35u;
    h ^= h >> 16;
    return h;
}

// First slot of a key's probe sequence: its home slot (hash & cap_mask) rounded
// down to the start of the home group.  Probing then runs over consecutive slots.
// A key is stored within this many slots of the start of its home group (or
// anywhere, for a smaller table): inserts that find no free slot in that
// window flag LAT_ERR_TABLE_FULL, so lookups stop after it.  At the load
// factors lat_hash_bytes gives (1/8 to 1/2 for ratios 2 to 8) probe
// sequences are a few slots long; only a table filled close to capacity
// reaches the limit.  It also bounds the work of a lookup in a table that
// lat_hash_build did not fill.
constexpr uint32_t kMaxProbeSlots = 4096;
__device__ __forceinline__ uint32_t probe_window(uint32_t cap_mask) {
    return cap_mask < kMaxProbeSlots - 1 ? cap_mask + 1 : kMaxProbeSlots;
}

// The home slot is the hash of the key's z-brick, the key with the low two bits
// of its z field cleared: the (up to) 4 cells of one z-run share a probe
// sequence, so a lookup of the z-neighbours of a cell (the 3 offsets of one
// kernel column) reads one group (two when the run crosses a brick edge).
__device__ __forceinline__ uint32_t probe_start(uint64_t key, uint32_t cap_mask) {
    return slot_hash(key & ~uint64_t(3)) & cap_mask & ~uint32_t(kGroupSlots - 1);
}

__device__ __forceinline__ uint64_t ptx_globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}


// Programmatic dependent launch.  Kernels started with launch_pdl may be
// scheduled while the previous kernel on the stream is still running:
// pdl_wait() blocks until that grid has completed and its memory is visible,
// and must come before the first global access; pdl_trigger() lets the next
// grid on the stream be scheduled now (its blocks then sit in their own
// pdl_wait()).  Both are no-ops for a kernel launched the ordinary way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
    pdl_wait();
    pdl_trigger();
}

__device__ __forceinline__ void flag(int32_t *d_status, int32_t bits) {
    if (d_status) atomicOr(d_status, bits);
}

// floor division by a positive divisor
__device__ __forceinline__ int floordiv(int a, int b) {
    int q = a / b;
    return (a % b != 0 && a < 0) ? q - 1 : q;
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__half> {
    static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
    static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

}  // namespace lat

// Host-side error plumbing.
#define LAT_CUDA_TRY(expr)                                   \
    do {                                                     \
        cudaError_t _e = (expr);                             \
        if (_e != cudaSuccess) return LAT_ERR_CUDA;          \
    } while (0)

namespace lat {
// SM count of the current device (looked up once per device).
inline int num_sms() {
    constexpr int kMaxDev = 64;
    static int cached[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
    if (cached[dev] <= 0) {
        int n = 148;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n;
    }
    return cached[dev];
}
inline bool pow2(uint64_t v) { return v && !(v & (v - 1)); }

// Limit of every barrier wait in the tensor-core kernels (lat_set_wait_limit_ns):
// one process-wide value, read when a kernel is launched.
inline std::atomic<uint64_t> &wait_limit_store() {
    static std::atomic<uint64_t> v{2000000000ull};
    return v;
}
inline uint64_t wait_limit_ns() { return wait_limit_store().load(std::memory_order_relaxed); }

// launch_pdl: launch with programmatic stream serialization: the kernel may be scheduled
// as soon as the previous kernel on `s` has triggered (every kernel of the
// library calls pdl_enter() first), so its launch latency overlaps that
// kernel's tail instead of following it.  Ordering is unchanged: the kernel's
// pdl_wait() returns only once the previous grid has completed.
template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A &&...args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// Fills n 32-bit words at p with v: a kernel rather than cudaMemsetAsync, so
// that it joins the programmatic launch chain of the kernels around it.
template <int = 0>
__global__ void __launch_bounds__(256) fill_u32_kernel(uint32_t *__restrict__ p, int64_t n, uint32_t v) {
    pdl_enter();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t i0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    const int64_t n4 = reinterpret_cast<uintptr_t>(p) % 16 == 0 ? n / 4 : 0;
    const uint4 v4 = make_uint4(v, v, v, v);
    for (int64_t i = i0; i < n4; i += stride) reinterpret_cast<uint4 *>(p)[i] = v4;
    for (int64_t i = 4 * n4 + i0; i < n; i += stride) p[i] = v;
}
inline cudaError_t fill_u32(void *p, int64_t n, uint32_t v, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int64_t want = (n / 4 + 255) / 256 + 1, cap = int64_t(num_sms()) * 8;
    return launch_pdl(fill_u32_kernel<0>, dim3(unsigned(want < cap ? want : cap)), dim3(256), 0, s,
                      static_cast<uint32_t *>(p), n, v);
}

// Up to kMaxFills regions of 32-bit words, each filled with its own value by
// one launch (fill_list): the zero / -1 initialisations an entry point needs
// cost one kernel instead of one each.
constexpr int kMaxFills = 6;
struct FillList {
    uint32_t *p[kMaxFills];
    int64_t n[kMaxFills];
    uint32_t v[kMaxFills];
    int count = 0;
    void add(void *ptr, int64_t words, uint32_t value) {
        if (words <= 0 || count >= kMaxFills) return;
        p[count] = static_cast<uint32_t *>(ptr);
        n[count] = words;
        v[count] = value;
        ++count;
    }
};
template <int = 0>
__global__ void __launch_bounds__(256) fill_list_kernel(FillList f) {
    pdl_enter();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t i0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
#pragma unroll
    for (int r = 0; r < kMaxFills; ++r) {
        if (r >= f.count) break;
        uint32_t *p = f.p[r];
        const int64_t n = f.n[r];
        const uint32_t v = f.v[r];
        const int64_t n4 = reinterpret_cast<uintptr_t>(p) % 16 == 0 ? n / 4 : 0;
        const uint4 v4 = make_uint4(v, v, v, v);
        for (int64_t i = i0; i < n4; i += stride) reinterpret_cast<uint4 *>(p)[i] = v4;
        for (int64_t i = 4 * n4 + i0; i < n; i += stride) p[i] = v;
    }
}
inline cudaError_t fill_list(const FillList &f, cudaStream_t s) {
    if (f.count == 0) return cudaSuccess;
    int64_t words = 0;
    for (int r = 0; r < f.count; ++r) words = f.n[r] > words ? f.n[r] : words;
    const int64_t want = (words / 4 + 255) / 256 + 1, cap = int64_t(num_sms()) * 8;
    return launch_pdl(fill_list_kernel<0>, dim3(unsigned(want < cap ? want : cap)), dim3(256), 0, s, f);
}

// A side stream for independent chains of small kernels inside one entry
// point: fork() makes it wait for everything enqueued on `s` so far, join()
// makes `s` wait for everything enqueued on it since.  One side stream and one
// pair of events per host thread and device, created on first use (make that
// first call outside a stream capture); the event fork / join also works while
// `s` is being captured into a graph.
struct SideStream {
    cudaStream_t side = nullptr;
    cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
};
inline cudaError_t side_stream(SideStream *&out) {
    constexpr int kMaxDev = 64;
    thread_local SideStream per_dev[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    SideStream &ss = per_dev[dev];
    if (!ss.side) {
        if ((e = cudaStreamCreateWithFlags(&ss.side, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&ss.fork_ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&ss.join_ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    out = &ss;
    return cudaSuccess;
}
inline cudaError_t side_fork(SideStream &ss, cudaStream_t s) {
    cudaError_t e = cudaEventRecord(ss.fork_ev, s);
    return e == cudaSuccess ? cudaStreamWaitEvent(ss.side, ss.fork_ev, 0) : e;
}
inline cudaError_t side_join(SideStream &ss, cudaStream_t s) {
    cudaError_t e = cudaEventRecord(ss.join_ev, ss.side);
    return e == cudaSuccess ? cudaStreamWaitEvent(s, ss.join_ev, 0) : e;
}

// CTAs of a persistent kernel that can be resident at once on the current device.
// The kernels are compiled with __launch_bounds__(threads, max_per_sm), so
// registers admit max_per_sm CTAs; shared memory admits
// smem_per_sm / (dynamic + static + per-block reserve); tensor memory (512
// columns per SM) admits 512 / tmem_cols.  (The runtime occupancy query
// under-reports here, so the limit is computed from the device attributes.)
// Also raises the kernel's dynamic shared-memory limit and asks for the
// largest carveout.  Returns 0 on error.
template <typename K>
inline int64_t persistent_grid_uncached(K kern, uint32_t smem, int tmem_cols, int max_per_sm) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) return 0;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return 0;
    int smem_sm = 0, reserve = 0;
    if (cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserve, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
        return 0;
    int per_sm = max_per_sm;
    const size_t per_cta = size_t(smem) + fa.sharedSizeBytes + size_t(reserve);
    if (int(smem_sm / per_cta) < per_sm) per_sm = int(smem_sm / per_cta);
    if (tmem_cols > 0 && per_sm > 512 / tmem_cols) per_sm = 512 / tmem_cols;
    if (per_sm < 1) return 0;
    return int64_t(per_sm) * num_sms();
}

// Per-device cache of one kernel's persistent grid; instantiate once per kernel
// (the Tag makes every kernel's cache distinct).  The first call on a device
// sets the kernel's attributes there.
template <typename Tag>
struct GridCache {
    template <typename K>
    static int64_t get(K kern, uint32_t smem, int tmem_cols, int max_per_sm) {
        constexpr int kMaxDev = 64;
        static int64_t cached[kMaxDev] = {};
        static std::mutex mu;
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 0;
        std::lock_guard<std::mutex> lock(mu);
        if (cached[dev] <= 0) cached[dev] = persistent_grid_uncached(kern, smem, tmem_cols, max_per_sm);
        return cached[dev];
    }
};
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Carves consecutive 256-byte aligned sub-buffers out of a caller workspace.
struct Carver {
    char *base;
    size_t used = 0;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <typename T> T *take(size_t count) {
        used = align_up(used, 256);
        T *p = base ? reinterpret_cast<T *>(base + used) : nullptr;
        used += count * sizeof(T);
        return p;
    }
};
}  // namespace lat
