// GPU open-addressing hash of packed coordinate keys (lat_hash_bytes, lat_hash_build).
//
// Torch Lattice docs, "Migrating from TorchSparse": hashing is one of the CUDA
// kernels of the library ("What remains familiar") and its capacity knob is
// torch_lattice.backends.hash_rsv_ratio ("Backend and configuration
// differences").  Design: 64-byte groups of 4 slots (4 keys, then 4 rows),
// 32-bit mixing hash of the key's z-brick (4 consecutive z cells share a home
// group, see probe_start), probing from the start of the home group over
// consecutive slots (at most kMaxProbeSlots of them), 64-bit atomicCAS to claim a
// slot and an unsigned atomicMin on the row so that duplicates keep the lowest
// row deterministically.
#include "common.cuh"

namespace lat {

__global__ void __launch_bounds__(256) hash_insert_kernel(const int4 *__restrict__ coords, int64_t n,
                                                          SlotGroup *__restrict__ groups, uint32_t cap_mask,
                                                          int32_t *d_status) {
    pdl_enter();
    int32_t bad = 0;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int4 c = __ldg(coords + i);
        uint64_t key;
        if (!pack_key(c.x, c.y, c.z, c.w, key)) {
            bad |= LAT_ERR_COORD_RANGE;
            continue;
        }
        uint32_t s = probe_start(key, cap_mask);
        bool placed = false;
        const uint32_t window = probe_window(cap_mask);
        for (uint32_t probe = 0; probe < window; ++probe) {
            // the CAS returns the slot's key: empty (now ours), ours (a duplicate) or another key
            unsigned long long *kp = &groups[s / kGroupSlots].key[s % kGroupSlots];
            const unsigned long long cur = atomicCAS(kp, (unsigned long long)kEmptyKey, (unsigned long long)key);
            if (cur == kEmptyKey || cur == key) {
                atomicMin(&groups[s / kGroupSlots].row[s % kGroupSlots], unsigned(i));
                if (cur == key) bad |= LAT_ERR_DUPLICATE;
                placed = true;
                break;
            }
            s = (s + 1) & cap_mask;
        }
        if (!placed) bad |= LAT_ERR_TABLE_FULL;
    }
    if (bad) flag(d_status, bad);
}

}  // namespace lat

extern "C" size_t lat_hash_bytes(int64_t n, float rsv_ratio) {
    if (n < 0 || !(rsv_ratio >= 1.0f) || n > (int64_t(1) << 31)) return 0;
    double want = double(rsv_ratio) * double(n);
    uint64_t cap = 64;
    while (double(cap) < want) cap <<= 1;
    if (cap > (uint64_t(1) << 31)) return 0;  // slot indices are 32-bit in the query kernels
    return size_t(cap) * lat::kSlotBytes;
}

extern "C" lat_status lat_hash_build(const int32_t *coords, int64_t n, void *table, size_t table_bytes,
                                     int32_t *d_status, lat_stream stream) {
    using namespace lat;
    if (n < 0 || n >= (int64_t(1) << 31) || (n > 0 && !coords) || !table) return LAT_ERR_ARG;
    if (table_bytes % kSlotBytes || !pow2(table_bytes / kSlotBytes) || table_bytes / kSlotBytes < 64 ||
        table_bytes / kSlotBytes > (uint64_t(1) << 31))
        return LAT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(coords) % 16 || reinterpret_cast<uintptr_t>(table) % 64) return LAT_ERR_ARG;
    const uint64_t cap = table_bytes / kSlotBytes;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // all-ones keys mark empty slots; a fill kernel (not a memset) keeps the
    // clearing in the programmatic launch chain of the kernels around it
    LAT_CUDA_TRY(fill_u32(table, int64_t(table_bytes / 4), 0xFFFFFFFFu, s));
    if (n == 0) return LAT_OK;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    LAT_CUDA_TRY(launch_pdl(hash_insert_kernel, dim3(unsigned(blocks)), dim3(threads), 0, s,
                            reinterpret_cast<const int4 *>(coords), n, static_cast<SlotGroup *>(table),
                            uint32_t(cap - 1), d_status));
    LAT_CUDA_TRY(cudaGetLastError());
    return LAT_OK;
}
