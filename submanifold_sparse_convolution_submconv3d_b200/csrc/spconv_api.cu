// C ABI of the SubMConv3d library: validation, the map handle, dispatch.
#include <string>
#include <new>

#include "common.cuh"

struct spconv_map_s {
    spconv::MapData d;
};

namespace {

thread_local std::string g_last_error;
int64_t g_table_slots_override = 0;
int32_t g_tile_rows_override = 0;

spconv_status_t fail(spconv_status_t s, const std::string& msg) {
    g_last_error = msg;
    return s;
}

spconv_status_t fail_cuda(cudaError_t e, const char* where) {
    g_last_error = std::string(where) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return e == cudaErrorMemoryAllocation ? SPCONV_ERR_OOM : SPCONV_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint64_t next_pow2(uint64_t v) {
    uint64_t p = 1;
    while (p < v) p <<= 1;
    return p;
}

}  // namespace

namespace spconv {
void set_last_error(const std::string& msg) { g_last_error = msg; }
}  // namespace spconv

extern "C" {

const char* spconv_last_error(void) { return g_last_error.c_str(); }

spconv_status_t spconv_debug_set_table_slots(int64_t slots) {
    if (slots < 0 || (slots & (slots - 1)) != 0) return fail(SPCONV_ERR_INVALID_ARG, "slots must be 0 or a power of two");
    g_table_slots_override = slots;
    return SPCONV_OK;
}

spconv_status_t spconv_map_tile_rows(spconv_map_t map, int32_t* rows) {
    if (!map || !rows) return fail(SPCONV_ERR_INVALID_ARG, "null map or rows");
    *rows = map->d.tile_rows;
    return SPCONV_OK;
}

spconv_status_t spconv_debug_set_tile_rows(int32_t rows) {
    if (rows < 0 || rows > spconv::kTileRows) return fail(SPCONV_ERR_INVALID_ARG, "rows must be in [0, 384]");
    g_tile_rows_override = rows;
    return SPCONV_OK;
}

spconv_status_t spconv_build_map(const int32_t* coords, int64_t n, const int32_t* extent, int32_t kernel_size,
                                 void* stream_, spconv_map_t* out_map) {
    g_last_error.clear();
    if (!out_map || !extent) return fail(SPCONV_ERR_INVALID_ARG, "null extent or out_map");
    if (kernel_size != 1 && kernel_size != 3) return fail(SPCONV_ERR_INVALID_ARG, "kernel_size must be 1 or 3");
    if (n < 0 || n >= (int64_t(1) << 31)) return fail(SPCONV_ERR_INVALID_ARG, "n must be in [0, 2^31)");
    for (int a = 0; a < 3; ++a)
        if (extent[a] < 1 || extent[a] > 65535) return fail(SPCONV_ERR_INVALID_ARG, "extent must be in [1, 65535]");
    if (n > 0 && (!coords || !aligned16(coords))) return fail(SPCONV_ERR_INVALID_ARG, "coords must be a 16-byte aligned device pointer");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);

    spconv_map_s* m = new (std::nothrow) spconv_map_s();
    if (!m) return fail(SPCONV_ERR_OOM, "host allocation failed");
    m->d.n = n;
    m->d.kernel_size = kernel_size;
    for (int a = 0; a < 3; ++a) m->d.extent[a] = extent[a];
    cudaError_t e = cudaGetDevice(&m->d.device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&m->d.num_sms, cudaDevAttrMultiProcessorCount, m->d.device);
    if (e == cudaSuccess) e = cudaMalloc(&m->d.fwd_err, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemsetAsync(m->d.fwd_err, 0, sizeof(unsigned int), stream);
    if (e != cudaSuccess) {
        cudaFree(m->d.fwd_err);
        delete m;
        return fail_cuda(e, "spconv_build_map setup");
    }

    uint64_t slots = g_table_slots_override > 0 ? (uint64_t)g_table_slots_override
                                                : next_pow2(n * 2 > 64 ? (uint64_t)n * 2 : 64);
    unsigned long long* table = nullptr;
    spconv::BuildFlags* flags = nullptr;
    spconv::BuildFlags host_flags{};
    spconv_status_t status = SPCONV_OK;
    e = cudaMalloc(&table, slots * 16);
    if (e == cudaSuccess) e = cudaMalloc(&flags, sizeof(spconv::BuildFlags));
    if (e == cudaSuccess && kernel_size == 3 && n > 0) e = cudaMalloc(&m->d.nbr, (size_t)n * spconv::kVol3 * sizeof(int32_t));
    m->d.tile_rows = g_tile_rows_override > 0 ? g_tile_rows_override : spconv::choose_tile_rows(n, m->d.num_sms);
    const int64_t ntiles = spconv::num_tiles(n, m->d.tile_rows);
    const bool tiles = kernel_size == 3 && n > 0;
    if (e == cudaSuccess && tiles) e = cudaMalloc(&m->d.tile_counts, (size_t)ntiles * spconv::kTileCountStride * 4);
    if (e == cudaSuccess && tiles) e = cudaMalloc(&m->d.tile_off, (size_t)(ntiles + 2) * sizeof(int64_t));
    if (e == cudaSuccess)
        e = spconv::launch_build_map(coords, n, extent, kernel_size, table, slots, m->d.nbr, flags, stream);
    if (e == cudaSuccess && tiles)
        e = spconv::launch_tile_count(m->d.nbr, n, m->d.tile_rows, m->d.tile_counts, m->d.tile_off, stream);
    int64_t entry_stats[2] = {0, 0};  // grand total, largest tile
    if (e == cudaSuccess && tiles)
        e = cudaMemcpyAsync(entry_stats, m->d.tile_off + ntiles, sizeof(entry_stats), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_flags, flags, sizeof(host_flags), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    // Second phase (only if the map is valid): entry arrays of the tile metadata.
    // entry_stats and host_flags are read only after the synchronisation above.
    if (e == cudaSuccess && tiles && host_flags.err == 0) {
        const int64_t total_entries = entry_stats[0];
        m->d.tile_entries = total_entries;
        m->d.tile_max_entries = entry_stats[1];
        const size_t ne = total_entries > 0 ? (size_t)total_entries : 1;
        e = cudaMalloc(&m->d.pair_r, ne * sizeof(uint16_t));
        if (e == cudaSuccess) e = cudaMalloc(&m->d.pair_j, ne * sizeof(int32_t));
        if (e == cudaSuccess)
            e = spconv::launch_tile_fill(m->d.nbr, n, m->d.tile_rows, m->d.tile_counts, m->d.tile_off, m->d.pair_r,
                                         m->d.pair_j, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    if (e != cudaSuccess) {
        status = fail_cuda(e, "spconv_build_map");
    } else if (host_flags.err & spconv::kErrCoordRange) {
        status = fail(SPCONV_ERR_COORD_RANGE, "a coordinate is outside [0, extent) or a batch index outside [0, 65535]");
    } else if (host_flags.err & spconv::kErrDuplicate) {
        status = fail(SPCONV_ERR_DUPLICATE, "duplicate (b, x, y, z) coordinates");
    } else if (host_flags.err & spconv::kErrTableFull) {
        status = fail(SPCONV_ERR_TABLE_FULL, "hash table full");
    }
    cudaFree(table);
    cudaFree(flags);
    if (status != SPCONV_OK) {
        spconv_free(m);
        return status;
    }
    m->d.pairs = kernel_size == 3 ? (int64_t)host_flags.pairs : n;
    *out_map = m;
    return SPCONV_OK;
}

spconv_status_t spconv_free(spconv_map_t map) {
    if (!map) return SPCONV_OK;
    cudaFree(map->d.nbr);
    cudaFree(map->d.fwd_err);
    cudaFree(map->d.tile_counts);
    cudaFree(map->d.tile_off);
    cudaFree(map->d.pair_r);
    cudaFree(map->d.pair_j);
    delete map;
    return SPCONV_OK;
}

spconv_status_t spconv_map_info(spconv_map_t map, int64_t* n, int32_t* kernel_size, int64_t* pairs,
                                const int32_t** nbr_dev) {
    if (!map) return fail(SPCONV_ERR_INVALID_ARG, "null map");
    if (n) *n = map->d.n;
    if (kernel_size) *kernel_size = map->d.kernel_size;
    if (pairs) *pairs = map->d.pairs;
    if (nbr_dev) *nbr_dev = map->d.nbr;
    return SPCONV_OK;
}

spconv_status_t spconv_map_check(spconv_map_t map, void* stream_) {
    if (!map) return fail(SPCONV_ERR_INVALID_ARG, "null map");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    unsigned int err = 0;
    cudaError_t e = cudaMemcpyAsync(&err, map->d.fwd_err, sizeof(err), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && err) e = cudaMemsetAsync(map->d.fwd_err, 0, sizeof(unsigned int), stream);
    if (e != cudaSuccess) return fail_cuda(e, "spconv_map_check");
    if (err & spconv::kFwdErrTimeout) return fail(SPCONV_ERR_TIMEOUT, "a device-side wait in a forward kernel gave up");
    return SPCONV_OK;
}

spconv_status_t spconv_subm_forward_algo(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                         const void* w, const void* bias, void* out, int32_t cout,
                                         spconv_algo_t algo, void* stream_) {
    g_last_error.clear();
    if (!map) return fail(SPCONV_ERR_INVALID_ARG, "null map");
    if (dtype != SPCONV_F32 && dtype != SPCONV_BF16) return fail(SPCONV_ERR_INVALID_ARG, "dtype must be SPCONV_F32 or SPCONV_BF16");
    if (algo != SPCONV_ALGO_AUTO && algo != SPCONV_ALGO_SIMT && algo != SPCONV_ALGO_TCGEN05)
        return fail(SPCONV_ERR_INVALID_ARG, "unknown algo");
    if (cin < 1 || cout < 1) return fail(SPCONV_ERR_INVALID_ARG, "cin and cout must be >= 1");
    if (dtype == SPCONV_BF16 && (cin % 16 != 0 || cout % 16 != 0))
        return fail(SPCONV_ERR_UNSUPPORTED, "bf16 needs cin and cout to be multiples of 16");
    if (map->d.n == 0) return SPCONV_OK;
    {   // the map's buffers live on its device: launch there only
        int dev = -1;
        const cudaError_t de = cudaGetDevice(&dev);
        if (de != cudaSuccess) return fail_cuda(de, "spconv_subm_forward");
        if (dev != map->d.device)
            return fail(SPCONV_ERR_INVALID_ARG, "the current CUDA device is not the device the map was built on");
    }
    if (!x || !w || !out) return fail(SPCONV_ERR_INVALID_ARG, "null x, w or out");
    if (!aligned16(x) || !aligned16(w) || !aligned16(out) || (bias && !aligned16(bias)))
        return fail(SPCONV_ERR_INVALID_ARG, "x, w, bias and out must be 16-byte aligned");
    const size_t esz = dtype == SPCONV_F32 ? 4 : 2;
    {   // out must not overlap x
        const char* xb = static_cast<const char*>(x);
        const char* ob = static_cast<const char*>(out);
        const size_t xbytes = (size_t)map->d.n * cin * esz, obytes = (size_t)map->d.n * cout * esz;
        if (ob < xb + xbytes && xb < ob + obytes) return fail(SPCONV_ERR_INVALID_ARG, "out overlaps x");
    }
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (algo == SPCONV_ALGO_TCGEN05 && dtype != SPCONV_BF16)
        return fail(SPCONV_ERR_UNSUPPORTED, "the tcgen05 kernel is bf16 only");
    if (dtype == SPCONV_BF16 && algo != SPCONV_ALGO_SIMT) {
        cudaError_t ce = cudaSuccess;
        spconv_status_t s = spconv::launch_forward_tcgen05(map->d, x, cin, w, bias, out, cout, stream, &ce);
        if (s == SPCONV_ERR_CUDA) return fail_cuda(ce, "tcgen05 forward");
        if (s == SPCONV_OK) return SPCONV_OK;
        // The tensor-core kernel takes cout % 64 == 0; AUTO runs other bf16 shapes
        // on the CUDA-core kernel.
        if (algo == SPCONV_ALGO_TCGEN05)
            return fail(s, "tcgen05 forward does not take this shape (cout % 64 != 0, cin % 16 != 0, or the tile lists "
                           "do not fit shared memory)");
    }
    cudaError_t e = spconv::launch_forward_simt(map->d, dtype, x, cin, w, bias, out, cout, stream);
    if (e != cudaSuccess) return fail_cuda(e, "simt forward");
    return SPCONV_OK;
}

spconv_status_t spconv_subm_forward(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                    const void* w, const void* bias, void* out, int32_t cout, void* stream) {
    return spconv_subm_forward_algo(map, dtype, x, cin, w, bias, out, cout, SPCONV_ALGO_AUTO, stream);
}

}  // extern "C"
