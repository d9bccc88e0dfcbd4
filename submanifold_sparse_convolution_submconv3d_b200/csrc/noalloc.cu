// Neighbour-map build that allocates no device memory.
//
// spconv_build_map allocates its hash table and flags with cudaMalloc and frees
// them with cudaFree.  Some callers cannot do that: code that runs while another
// component owns the device memory budget (a framework's caching allocator, a
// fixed arena reserved up front), and latency-critical loops, because cudaFree
// synchronises the whole device and cudaMalloc can stall work on other streams.
// spconv_build_neighbor_map_noalloc serves them: the caller passes the output
// buffer, and the hash table and error flags live in the file-scope array below,
// which every GPU that loads this library holds until the process exits.
#include <string>

#include "common.cuh"

namespace {

// Largest coordinate set this entry point accepts, and the table it needs
// (power of two >= 2n slots of 16 bytes, plus the flags).
constexpr int64_t kNoAllocMaxVoxels = int64_t(1) << 19;  // 524,288 voxels
constexpr uint64_t kNoAllocSlots = uint64_t(1) << 20;     // 16 MiB of table
constexpr size_t kNoAllocTableBytes = kNoAllocSlots * 16;
constexpr size_t kNoAllocBytes = kNoAllocTableBytes + 256;  // + BuildFlags, 256-byte aligned

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

spconv_status_t noalloc_fail(spconv_status_t s, const std::string& msg) {
    spconv::set_last_error(msg);
    return s;
}

// Device address of the scratch array on the current device.  In host code the
// array's name only stands in for it, so the address is asked of the runtime with
// the device current.  It is looked up on every call (the lookup allocates
// nothing): a cached address would go stale if the device's context were reset.
cudaError_t scratch_for_current_device(unsigned char** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = static_cast<unsigned char*>(p);
    return cudaSuccess;
}

}  // namespace

extern "C" {

spconv_status_t spconv_build_neighbor_map_noalloc(const int32_t* coords, int64_t n, const int32_t* extent,
                                                  int32_t* nbr_out, int64_t* pairs_out, void* stream_) {
    spconv::set_last_error(std::string());
    if (!extent) return noalloc_fail(SPCONV_ERR_INVALID_ARG, "null extent");
    if (n < 0) return noalloc_fail(SPCONV_ERR_INVALID_ARG, "n must be >= 0");
    if (n > kNoAllocMaxVoxels)
        return noalloc_fail(SPCONV_ERR_UNSUPPORTED,
                            "n exceeds the 524288-voxel limit of the allocation-free build (use spconv_build_map)");
    for (int a = 0; a < 3; ++a)
        if (extent[a] < 1 || extent[a] > 65535)
            return noalloc_fail(SPCONV_ERR_INVALID_ARG, "extent must be in [1, 65535]");
    if (n > 0 && (!coords || (reinterpret_cast<uintptr_t>(coords) & 15u) != 0))
        return noalloc_fail(SPCONV_ERR_INVALID_ARG, "coords must be a 16-byte aligned device pointer");
    if (n > 0 && (!nbr_out || (reinterpret_cast<uintptr_t>(nbr_out) & 3u) != 0))
        return noalloc_fail(SPCONV_ERR_INVALID_ARG, "nbr_out must be a 4-byte aligned device pointer");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);

    unsigned char* scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess)
        return noalloc_fail(SPCONV_ERR_CUDA, std::string("scratch lookup: ") + cudaGetErrorString(e));
    auto* table = reinterpret_cast<unsigned long long*>(scratch);
    auto* flags = reinterpret_cast<spconv::BuildFlags*>(scratch + kNoAllocTableBytes);
    // Table and flags are cleared on the stream before use (the array keeps the
    // previous call's contents).  Slots: power of two >= 2n, at most the array.
    uint64_t slots = 64;
    while (slots < (uint64_t)n * 2) slots <<= 1;
    e = spconv::launch_build_map(coords, n, extent, 3, table, slots, nbr_out, nullptr, flags, stream);
    spconv::BuildFlags host_flags{};
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_flags, flags, sizeof(host_flags), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return noalloc_fail(SPCONV_ERR_CUDA, std::string("build: ") + cudaGetErrorString(e));
    if (host_flags.err & spconv::kErrCoordRange)
        return noalloc_fail(SPCONV_ERR_COORD_RANGE, "a coordinate is outside [0, extent) or a batch index outside [0, 65535]");
    if (host_flags.err & spconv::kErrDuplicate)
        return noalloc_fail(SPCONV_ERR_DUPLICATE, "duplicate (b, x, y, z) coordinates");
    if (host_flags.err & spconv::kErrTableFull) return noalloc_fail(SPCONV_ERR_TABLE_FULL, "hash table full");
    if (pairs_out) *pairs_out = n > 0 ? (int64_t)host_flags.pairs : 0;
    return SPCONV_OK;
}

}  // extern "C"
