// C ABI of the SubMConv3d library: validation, the map handle, dispatch.
//
// Device memory of the maps comes from one stream-ordered memory pool per device
// that the library owns (cudaMallocFromPoolAsync on the build's stream).  The pool
// keeps freed memory for reuse, so a map build after the first one maps no new
// memory and never synchronises the device; the build synchronises its stream
// once, at the end, to read back the device error flags.
#include <atomic>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"

struct spconv_map_s {
    spconv::MapData d;
    std::atomic<int64_t> launches[SPCONV_KERNEL_KINDS] = {};  // forward launches per kernel family
    std::vector<void*> owned;                                  // pool allocations the map owns
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

// The library's memory pool of device `dev`, created on first use.  Its release
// threshold is the maximum, so memory freed to it stays mapped for later builds.
cudaError_t device_pool(int dev, cudaMemPool_t* out) {
    static std::mutex mu;
    static std::vector<cudaMemPool_t> pools;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0) return cudaErrorInvalidDevice;
    if (dev >= (int)pools.size()) pools.resize((size_t)dev + 1, nullptr);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        cudaError_t e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        uint64_t threshold = ~0ull;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &threshold);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        pools[dev] = pool;
    }
    *out = pools[dev];
    return cudaSuccess;
}

// Stream-ordered allocations of one build: the map's own buffers and transient
// scratch, released on the build's stream.
struct BuildAlloc {
    cudaMemPool_t pool = nullptr;
    cudaStream_t stream = nullptr;
    std::vector<void*> scratch;
    cudaError_t err = cudaSuccess;

    template <typename T>
    T* get(size_t count, std::vector<void*>& owner) {
        if (err != cudaSuccess) return nullptr;
        void* p = nullptr;
        err = cudaMallocFromPoolAsync(&p, count > 0 ? count * sizeof(T) : 16, pool, stream);
        if (err != cudaSuccess) return nullptr;
        owner.push_back(p);
        return static_cast<T*>(p);
    }
    template <typename T>
    T* temp(size_t count) { return get<T>(count, scratch); }
    void release_scratch() {
        for (void* p : scratch) cudaFreeAsync(p, stream);
        scratch.clear();
    }
};

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
    *rows = map->d.win_rows;
    return SPCONV_OK;
}

spconv_status_t spconv_debug_set_tile_rows(int32_t rows) {
    if (rows < 0 || rows > spconv::kWinMaxRows || rows % spconv::kWinCols != 0)
        return fail(SPCONV_ERR_INVALID_ARG, "rows must be 0 or a multiple of 16 in [16, 256]");
    g_tile_rows_override = rows;
    return SPCONV_OK;
}

spconv_status_t spconv_debug_set_ring_depths(int32_t a_slots, int32_t b_units) {
    const bool auto_ = a_slots == 0 && b_units == 0;
    if (!auto_ && (a_slots < 2 || a_slots > 8 || b_units < 4 || b_units > 32))
        return fail(SPCONV_ERR_INVALID_ARG, "a_slots must be in [2, 8] and b_units in [4, 32], or both 0");
    spconv::set_forced_ring_depths(a_slots, b_units);
    spconv::set_forced_gemm1_stages(a_slots);
    return SPCONV_OK;
}

spconv_status_t spconv_free(spconv_map_t map) {
    if (!map) return SPCONV_OK;
    int prev = -1;
    const bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
    if (map->d.device != prev) cudaSetDevice(map->d.device);
    // Kernels on any stream may still read the map: wait for the device, then
    // hand the memory back to the pool.
    cudaDeviceSynchronize();
    for (void* p : map->owned) cudaFreeAsync(p, nullptr);
    if (have_prev && map->d.device != prev) cudaSetDevice(prev);
    delete map;
    return SPCONV_OK;
}

}  // extern "C"

extern "C" {

spconv_status_t spconv_build_map_ex(const int32_t* coords, int64_t n, const int32_t* extent, int32_t kernel_size,
                                    uint32_t flags_, void* stream_, spconv_map_t* out_map) {
    g_last_error.clear();
    if (!out_map || !extent) return fail(SPCONV_ERR_INVALID_ARG, "null extent or out_map");
    if (kernel_size != 1 && kernel_size != 3) return fail(SPCONV_ERR_INVALID_ARG, "kernel_size must be 1 or 3");
    if (n < 0 || n >= (int64_t(1) << 31)) return fail(SPCONV_ERR_INVALID_ARG, "n must be in [0, 2^31)");
    if (flags_ & ~(uint32_t)(SPCONV_MAP_FLIP_KERNEL | SPCONV_MAP_SORTED_KEYS | SPCONV_MAP_HASH_TABLE |
                             SPCONV_MAP_SHORT_TILES))
        return fail(SPCONV_ERR_INVALID_ARG, "unknown map flag");
    if ((flags_ & SPCONV_MAP_SORTED_KEYS) && (flags_ & SPCONV_MAP_HASH_TABLE))
        return fail(SPCONV_ERR_INVALID_ARG, "SORTED_KEYS and HASH_TABLE exclude each other");
    for (int a = 0; a < 3; ++a)
        if (extent[a] < 1 || extent[a] > 65535) return fail(SPCONV_ERR_INVALID_ARG, "extent must be in [1, 65535]");
    spconv::MapBuildOpts opts;
    opts.flip = (flags_ & SPCONV_MAP_FLIP_KERNEL) != 0;
    const bool sorted_fits = spconv::sorted_key_bits(extent) <= 62;
    if ((flags_ & SPCONV_MAP_SORTED_KEYS) && !sorted_fits)
        return fail(SPCONV_ERR_UNSUPPORTED, "sorted-key build: 16 batch bits plus the extents' bits exceed 62");
    // Neither dictionary forced: the hash table (measured on B200 with the probes
    // batched: faster than the sorted keys on 0.2 M and 2.2 M voxels alike).
    opts.sorted = (flags_ & SPCONV_MAP_SORTED_KEYS) != 0;
    if (n > 0 && (!coords || !aligned16(coords))) return fail(SPCONV_ERR_INVALID_ARG, "coords must be a 16-byte aligned device pointer");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);

    spconv_map_s* m = new (std::nothrow) spconv_map_s();
    if (!m) return fail(SPCONV_ERR_OOM, "host allocation failed");
    spconv::MapData& d = m->d;
    d.n = n;
    d.kernel_size = kernel_size;
    d.flags = flags_;
    for (int a = 0; a < 3; ++a) d.extent[a] = extent[a];
    BuildAlloc al;
    al.stream = stream;
    cudaError_t e = cudaGetDevice(&d.device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, d.device);
    if (e == cudaSuccess) e = device_pool(d.device, &al.pool);
    if (e != cudaSuccess) {
        delete m;
        return fail_cuda(e, "spconv_build_map setup");
    }

    // Every size below follows from n, so all buffers are requested up front and
    // the build needs a single synchronisation at its end.
    d.win_rows = g_tile_rows_override > 0
                     ? g_tile_rows_override
                     : spconv::choose_win_rows(n, d.num_sms, (flags_ & SPCONV_MAP_SHORT_TILES) != 0);
    d.win_tiles = (n + d.win_rows - 1) / d.win_rows;
    d.npad = d.win_tiles * d.win_rows;
    const bool k3 = kernel_size == 3 && n > 0;
    const uint64_t slots = g_table_slots_override > 0 ? (uint64_t)g_table_slots_override
                                                      : next_pow2(n * 2 > 64 ? (uint64_t)n * 2 : 64);
    d.fwd_err = al.get<unsigned int>(1, m->owned);
    d.sched = al.get<uint32_t>(spconv::kSchedSlots, m->owned);
    auto* flags = al.temp<spconv::BuildFlags>(1);
    spconv::BuildFlags host_flags{};
    auto* table = opts.sorted ? nullptr : al.temp<unsigned long long>(slots * 2);
    uint32_t* keys[2] = {nullptr, nullptr};
    int32_t* vals[2] = {nullptr, nullptr};
    uint32_t* hist = nullptr;
    if (k3 || (opts.sorted && n > 0)) {
        vals[1] = al.temp<int32_t>((size_t)n);
        vals[0] = al.temp<int32_t>((size_t)n);
        hist = al.temp<uint32_t>((size_t)spconv::radix_hist_words(n));
    }
    if (opts.sorted && n > 0) {
        // the sorted dictionary reuses the row sort's value and count buffers
        opts.skeys[0] = al.temp<uint64_t>((size_t)n);
        opts.skeys[1] = al.temp<uint64_t>((size_t)n);
        opts.svals[0] = vals[0];
        opts.svals[1] = vals[1];
        opts.hist = hist;
    }
    if (k3) {
        d.nbr = al.get<int32_t>((size_t)n * spconv::kVol3, m->owned);
        d.perm = al.get<int32_t>((size_t)n, m->owned);
        d.nbr_t = al.get<int32_t>((size_t)d.npad * spconv::kVol3, m->owned);
        d.win_jobs = al.get<uint32_t>((size_t)d.win_tiles * spconv::kWinJobStride, m->owned);
        d.idx_off = al.get<int64_t>((size_t)d.win_tiles + 1, m->owned);
        d.win_order = al.get<int32_t>((size_t)d.win_tiles, m->owned);
        // a tile's stream holds at most its rows for each of the 27 offsets
        d.idx_stream = al.get<int32_t>((size_t)d.npad * spconv::kVol3, m->owned);
        keys[0] = al.temp<uint32_t>((size_t)n);
        keys[1] = al.temp<uint32_t>((size_t)n);
    }
    e = al.err;
    if (e == cudaSuccess) e = cudaMemsetAsync(d.fwd_err, 0, sizeof(unsigned int), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(d.sched, 0, spconv::kSchedSlots * sizeof(uint32_t), stream);
    if (e == cudaSuccess)
        e = spconv::launch_build_map(coords, n, extent, kernel_size, table, slots, d.nbr, keys[0], flags, stream,
                                     opts);
    if (e == cudaSuccess && k3) {
        // rows sorted by the Gray rank of their neighbour mask (26 bits); the
        // first pass takes the row indices as values
        int which = 0;
        e = spconv::radix_sort_pairs(keys, nullptr, vals, n, 26, hist, &which, stream);
        if (e == cudaSuccess)
            e = spconv::launch_win_meta(d.nbr, vals[which], n, d.win_rows, d.win_tiles, d.npad, d.perm, d.nbr_t,
                                        d.win_jobs, d.idx_off, d.idx_stream, flags, stream);
        // the tile claim order: tiles sorted (stably) by descending estimated cost;
        // the row sort's buffers are free again and hold at least `tiles` entries
        if (e == cudaSuccess) e = spconv::launch_win_cost(d.win_jobs, d.win_tiles, keys[0], stream);
        int which_t = 0;
        if (e == cudaSuccess) e = spconv::radix_sort_pairs(keys, nullptr, vals, d.win_tiles, 9, hist, &which_t, stream);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(d.win_order, vals[which_t], (size_t)d.win_tiles * sizeof(int32_t),
                                cudaMemcpyDeviceToDevice, stream);
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_flags, flags, sizeof(host_flags), cudaMemcpyDeviceToHost, stream);
    al.release_scratch();
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    spconv_status_t status = SPCONV_OK;
    if (e != cudaSuccess) {
        status = fail_cuda(e, "spconv_build_map");
    } else if (host_flags.err & spconv::kErrCoordRange) {
        status = fail(SPCONV_ERR_COORD_RANGE, "a coordinate is outside [0, extent) or a batch index outside [0, 65535]");
    } else if (host_flags.err & spconv::kErrDuplicate) {
        status = fail(SPCONV_ERR_DUPLICATE, "duplicate (b, x, y, z) coordinates");
    } else if (host_flags.err & spconv::kErrTableFull) {
        status = fail(SPCONV_ERR_TABLE_FULL, "hash table full");
    } else if (host_flags.err & spconv::kErrInternal) {
        status = fail(SPCONV_ERR_CUDA, "internal error: a metadata bound did not hold");
    }
    if (status != SPCONV_OK) {
        spconv_free(m);
        return status;
    }
    d.pairs = kernel_size == 3 ? (int64_t)host_flags.pairs : n;
    d.win_spans = (int64_t)host_flags.spans;
    d.win_span_cols = (int64_t)host_flags.span_cols;
    d.max_tile_cols = (int64_t)host_flags.max_tile_cols;
    *out_map = m;
    return SPCONV_OK;
}

spconv_status_t spconv_build_map(const int32_t* coords, int64_t n, const int32_t* extent, int32_t kernel_size,
                                 void* stream, spconv_map_t* out_map) {
    return spconv_build_map_ex(coords, n, extent, kernel_size, SPCONV_MAP_DEFAULT, stream, out_map);
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

spconv_status_t spconv_map_stats(spconv_map_t map, spconv_map_stats_t* stats) {
    if (!map || !stats) return fail(SPCONV_ERR_INVALID_ARG, "null map or stats");
    stats->tiles = map->d.win_tiles;
    stats->rows_per_tile = map->d.win_rows;
    stats->spans = map->d.win_spans;
    stats->span_cols = map->d.win_span_cols;
    stats->perm_dev = map->d.perm;
    stats->nbr_t_dev = map->d.nbr_t;
    stats->jobs_dev = map->d.win_jobs;
    stats->job_stride = spconv::kWinJobStride;
    stats->order_dev = map->d.win_order;
    return SPCONV_OK;
}

spconv_status_t spconv_map_check(spconv_map_t map, void* stream_) {
    if (!map) return fail(SPCONV_ERR_INVALID_ARG, "null map");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    unsigned int err = 0;
    cudaError_t e = cudaMemcpyAsync(&err, map->d.fwd_err, sizeof(err), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && err) e = cudaMemsetAsync(map->d.fwd_err, 0, sizeof(unsigned int), stream);
    // a forward that gave up may have left its work counter mid-count
    if (e == cudaSuccess && err && map->d.sched)
        e = cudaMemsetAsync(map->d.sched, 0, spconv::kSchedSlots * sizeof(uint32_t), stream);
    if (e != cudaSuccess) return fail_cuda(e, "spconv_map_check");
    if (err & spconv::kFwdErrTimeout) return fail(SPCONV_ERR_TIMEOUT, "a device-side wait in a forward kernel gave up");
    return SPCONV_OK;
}

spconv_status_t spconv_subm_forward_ex(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                       const void* w, const void* bias, void* out, int32_t cout,
                                       const spconv_epilogue_t* epi_, spconv_algo_t algo, void* stream_) {
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
    spconv::Epilogue epi;
    if (epi_) {
        if (epi_->act < SPCONV_ACT_NONE || epi_->act > SPCONV_ACT_GELU)
            return fail(SPCONV_ERR_INVALID_ARG, "unknown activation");
        epi.act = epi_->act;
        epi.residual = epi_->residual;
        epi.stats = epi_->stats;
        if (epi.residual) {
            if (!aligned16(epi.residual)) return fail(SPCONV_ERR_INVALID_ARG, "residual must be 16-byte aligned");
            const char* rb = static_cast<const char*>(epi.residual);
            const char* xb = static_cast<const char*>(x);
            const char* ob = static_cast<const char*>(out);
            const size_t rbytes = (size_t)map->d.n * cout * esz, xbytes = (size_t)map->d.n * cin * esz;
            if (rb < xb + xbytes && xb < rb + rbytes) return fail(SPCONV_ERR_INVALID_ARG, "residual overlaps x");
            if (rb != ob && rb < ob + rbytes && ob < rb + rbytes)
                return fail(SPCONV_ERR_INVALID_ARG, "residual partly overlaps out");
        }
        if (epi.stats && !aligned16(epi.stats)) return fail(SPCONV_ERR_INVALID_ARG, "stats must be 16-byte aligned");
    }
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (epi.stats) {
        const cudaError_t me = cudaMemsetAsync(epi.stats, 0, (size_t)2 * cout * sizeof(float), stream);
        if (me != cudaSuccess) return fail_cuda(me, "zeroing stats");
    }
    if (algo == SPCONV_ALGO_TCGEN05 && dtype != SPCONV_BF16)
        return fail(SPCONV_ERR_UNSUPPORTED, "the tcgen05 kernel is bf16 only");
    // AUTO: bf16 with cout % 64 == 0 runs on the tensor cores (kernel size 1 on
    // the weight-stationary GEMM when it takes the shape, else on the window
    // kernel); fp32 and other bf16 shapes on the CUDA-core kernel.  The choice
    // depends on the shape alone, and the map's launch counters record it.
    const bool tc_shape = dtype == SPCONV_BF16 && cout % 64 == 0;
    if (algo == SPCONV_ALGO_TCGEN05 || (algo == SPCONV_ALGO_AUTO && tc_shape)) {
        cudaError_t ce = cudaSuccess;
        if (map->d.kernel_size == 1) {
            const spconv_status_t g =
                spconv::launch_forward_gemm1(map->d, x, cin, w, bias, out, cout, epi, stream, &ce);
            if (g == SPCONV_ERR_CUDA) return fail_cuda(ce, "tcgen05 GEMM forward");
            if (g == SPCONV_OK) {
                map->launches[SPCONV_KERNEL_TCGEN05_GEMM].fetch_add(1);
                return SPCONV_OK;
            }
        }
        const spconv_status_t s = spconv::launch_forward_tcgen05(map->d, x, cin, w, bias, out, cout, epi, stream, &ce);
        if (s == SPCONV_ERR_CUDA) return fail_cuda(ce, "tcgen05 forward");
        if (s != SPCONV_OK)
            return fail(s, "the tcgen05 kernel does not take this shape (bf16 with cout % 64 == 0 and cin % 16 == 0)");
        map->launches[SPCONV_KERNEL_TCGEN05].fetch_add(1);
        return SPCONV_OK;
    }
    cudaError_t e = spconv::launch_forward_simt(map->d, dtype, x, cin, w, bias, out, cout, epi, stream);
    if (e != cudaSuccess) return fail_cuda(e, "simt forward");
    map->launches[SPCONV_KERNEL_SIMT].fetch_add(1);
    return SPCONV_OK;
}

spconv_status_t spconv_subm_forward_algo(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                         const void* w, const void* bias, void* out, int32_t cout,
                                         spconv_algo_t algo, void* stream) {
    return spconv_subm_forward_ex(map, dtype, x, cin, w, bias, out, cout, nullptr, algo, stream);
}

spconv_status_t spconv_subm_forward(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                    const void* w, const void* bias, void* out, int32_t cout, void* stream) {
    return spconv_subm_forward_ex(map, dtype, x, cin, w, bias, out, cout, nullptr, SPCONV_ALGO_AUTO, stream);
}

spconv_status_t spconv_map_launch_counts(spconv_map_t map, int64_t* counts, int32_t ncounts) {
    if (!map || !counts || ncounts < 1) return fail(SPCONV_ERR_INVALID_ARG, "null map or counts, or ncounts < 1");
    for (int32_t k = 0; k < ncounts; ++k) counts[k] = k < SPCONV_KERNEL_KINDS ? map->launches[k].load() : 0;
    return SPCONV_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ resampling
namespace spconv {
int64_t ds_scan_blocks(int64_t n);
int ds_key_bits(const int32_t coarse_extent[3]);
cudaError_t launch_ds_build(const int32_t* coords, int64_t n, const int32_t extent[3], int factor,
                            const int32_t coarse_extent[3], uint64_t* keys[2], int32_t* vals[2], uint32_t* hist,
                            uint32_t* counts, unsigned int* err, int32_t** srows_out, int4* coarse, int32_t* seg,
                            int32_t* parent, cudaStream_t stream);
cudaError_t launch_ds_amax(const int32_t* seg, const int32_t* srows, int64_t ncoarse, bool bf16, int c,
                           const void* x, void* out, cudaStream_t stream);
cudaError_t launch_upsample(const int32_t* parent, int64_t n, int64_t row_bytes, const void* xc, void* out,
                            cudaStream_t stream);
cudaError_t launch_subdivide(const int32_t* coords, int64_t n, const int32_t extent[3], int64_t row_bytes,
                             const void* x, int32_t* coords_out, void* x_out, unsigned int* err,
                             cudaStream_t stream);
}  // namespace spconv

struct spconv_downsample_s {
    int64_t n = 0, n_coarse = 0;
    int32_t factor = 1;
    int32_t coarse_extent[3] = {0, 0, 0};
    int32_t* coarse = nullptr;  // device int32 [n_coarse, 4]
    int32_t* parent = nullptr;  // device int32 [n]: coarse row of each fine row
    int32_t* seg = nullptr;     // device int32 [n_coarse + 1]: run starts in srows
    int32_t* srows = nullptr;   // device int32 [n]: fine rows sorted by coarse key (stable)
    int device = 0;
    std::vector<void*> owned;
};

namespace {

bool coords_arg_ok(const int32_t* coords, int64_t n, const int32_t* extent, int32_t max_extent, std::string* why) {
    if (!extent) return (*why = "null extent", false);
    if (n < 0 || n >= (int64_t(1) << 31)) return (*why = "n must be in [0, 2^31)", false);
    for (int a = 0; a < 3; ++a)
        if (extent[a] < 1 || extent[a] > max_extent)
            return (*why = "extent must be in [1, " + std::to_string(max_extent) + "]", false);
    if (n > 0 && (!coords || !aligned16(coords))) return (*why = "coords must be a 16-byte aligned device pointer", false);
    return true;
}

spconv_status_t rows_arg_check(spconv_dtype_t dtype, int32_t channels, const void* a, const void* b) {
    if (dtype != SPCONV_F32 && dtype != SPCONV_BF16) return fail(SPCONV_ERR_INVALID_ARG, "dtype must be F32 or BF16");
    if (channels < 1) return fail(SPCONV_ERR_INVALID_ARG, "channels must be >= 1");
    if (!a || !b || !aligned16(a) || !aligned16(b))
        return fail(SPCONV_ERR_INVALID_ARG, "feature pointers must be 16-byte aligned device pointers");
    return SPCONV_OK;
}

bool on_device(int dev) {
    int cur = -1;
    return cudaGetDevice(&cur) == cudaSuccess && cur == dev;
}

}  // namespace

extern "C" {

spconv_status_t spconv_downsample_free(spconv_downsample_t ds) {
    if (!ds) return SPCONV_OK;
    int prev = -1;
    const bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
    if (ds->device != prev) cudaSetDevice(ds->device);
    cudaDeviceSynchronize();
    for (void* p : ds->owned) cudaFreeAsync(p, nullptr);
    if (have_prev && ds->device != prev) cudaSetDevice(prev);
    delete ds;
    return SPCONV_OK;
}

spconv_status_t spconv_downsample_build(const int32_t* coords, int64_t n, const int32_t* extent, int32_t factor,
                                        void* stream_, spconv_downsample_t* out) {
    g_last_error.clear();
    std::string why;
    if (!out) return fail(SPCONV_ERR_INVALID_ARG, "null out");
    if (!coords_arg_ok(coords, n, extent, 65535, &why)) return fail(SPCONV_ERR_INVALID_ARG, why);
    if (factor < 1 || factor > 65535) return fail(SPCONV_ERR_INVALID_ARG, "factor must be in [1, 65535]");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    spconv_downsample_s* ds = new (std::nothrow) spconv_downsample_s();
    if (!ds) return fail(SPCONV_ERR_OOM, "host allocation failed");
    ds->n = n;
    ds->factor = factor;
    for (int a = 0; a < 3; ++a) ds->coarse_extent[a] = (extent[a] + factor - 1) / factor;
    BuildAlloc al;
    al.stream = stream;
    cudaError_t e = cudaGetDevice(&ds->device);
    if (e == cudaSuccess) e = device_pool(ds->device, &al.pool);
    if (e != cudaSuccess) {
        delete ds;
        return fail_cuda(e, "spconv_downsample_build setup");
    }
    if (n == 0) {
        *out = ds;
        return SPCONV_OK;
    }
    const int64_t blocks = spconv::ds_scan_blocks(n);
    uint64_t* keys[2] = {al.temp<uint64_t>((size_t)n), al.temp<uint64_t>((size_t)n)};
    int32_t* vals[2] = {al.temp<int32_t>((size_t)n), al.temp<int32_t>((size_t)n)};
    auto* hist = al.temp<uint32_t>((size_t)spconv::radix_hist_words(n));
    auto* counts = al.temp<uint32_t>((size_t)blocks + 1);
    auto* err = al.temp<unsigned int>(1);
    // the coarse set has at most n voxels; its exact size is known after the sync
    ds->coarse = al.get<int32_t>((size_t)n * 4, ds->owned);
    ds->seg = al.get<int32_t>((size_t)n + 1, ds->owned);
    ds->parent = al.get<int32_t>((size_t)n, ds->owned);
    e = al.err;
    if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(unsigned int), stream);
    int32_t* srows = nullptr;
    if (e == cudaSuccess)
        e = spconv::launch_ds_build(coords, n, extent, factor, ds->coarse_extent, keys, vals, hist, counts, err,
                                    &srows, reinterpret_cast<int4*>(ds->coarse), ds->seg, ds->parent, stream);
    uint32_t host[2] = {0, 0};
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host[0], counts + blocks, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host[1], err, 4, cudaMemcpyDeviceToHost, stream);
    // the sorted rows stay with the handle; the other scratch goes back to the pool
    if (srows) {
        for (auto& p : al.scratch)
            if (p == srows) p = nullptr;
        ds->owned.push_back(srows);
        ds->srows = srows;
    }
    for (void* p : al.scratch)
        if (p) cudaFreeAsync(p, stream);
    al.scratch.clear();
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    spconv_status_t status = SPCONV_OK;
    if (e != cudaSuccess) {
        status = fail_cuda(e, "spconv_downsample_build");
    } else if (host[1] & spconv::kErrCoordRange) {
        status = fail(SPCONV_ERR_COORD_RANGE, "a coordinate is outside [0, extent) or a batch index outside [0, 65535]");
    }
    if (status != SPCONV_OK) {
        spconv_downsample_free(ds);
        return status;
    }
    ds->n_coarse = host[0];
    *out = ds;
    return SPCONV_OK;
}

spconv_status_t spconv_downsample_info(spconv_downsample_t ds, int64_t* n_fine, int64_t* n_coarse,
                                       int32_t* coarse_extent, const int32_t** coarse_coords_dev,
                                       const int32_t** parent_dev) {
    if (!ds) return fail(SPCONV_ERR_INVALID_ARG, "null handle");
    if (n_fine) *n_fine = ds->n;
    if (n_coarse) *n_coarse = ds->n_coarse;
    if (coarse_extent)
        for (int a = 0; a < 3; ++a) coarse_extent[a] = ds->coarse_extent[a];
    if (coarse_coords_dev) *coarse_coords_dev = ds->coarse;
    if (parent_dev) *parent_dev = ds->parent;
    return SPCONV_OK;
}

spconv_status_t spconv_downsample_amax(spconv_downsample_t ds, spconv_dtype_t dtype, const void* x,
                                       int32_t channels, void* out, void* stream) {
    if (!ds) return fail(SPCONV_ERR_INVALID_ARG, "null handle");
    if (ds->n == 0) return SPCONV_OK;
    const spconv_status_t s = rows_arg_check(dtype, channels, x, out);
    if (s != SPCONV_OK) return s;
    if (!on_device(ds->device)) return fail(SPCONV_ERR_INVALID_ARG, "the current device is not the handle's device");
    const cudaError_t e = spconv::launch_ds_amax(ds->seg, ds->srows, ds->n_coarse, dtype == SPCONV_BF16, channels, x,
                                                 out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPCONV_OK : fail_cuda(e, "spconv_downsample_amax");
}

spconv_status_t spconv_upsample(spconv_downsample_t ds, spconv_dtype_t dtype, const void* x_coarse,
                                int32_t channels, void* out, void* stream) {
    if (!ds) return fail(SPCONV_ERR_INVALID_ARG, "null handle");
    if (ds->n == 0) return SPCONV_OK;
    const spconv_status_t s = rows_arg_check(dtype, channels, x_coarse, out);
    if (s != SPCONV_OK) return s;
    if (!on_device(ds->device)) return fail(SPCONV_ERR_INVALID_ARG, "the current device is not the handle's device");
    const int64_t row_bytes = (int64_t)channels * (dtype == SPCONV_BF16 ? 2 : 4);
    const cudaError_t e = spconv::launch_upsample(ds->parent, ds->n, row_bytes, x_coarse, out,
                                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPCONV_OK : fail_cuda(e, "spconv_upsample");
}

spconv_status_t spconv_subdivide(const int32_t* coords, int64_t n, const int32_t* extent, spconv_dtype_t dtype,
                                 const void* x, int32_t channels, int32_t* coords_out, void* x_out, void* stream_) {
    g_last_error.clear();
    std::string why;
    if (!coords_arg_ok(coords, n, extent, 32767, &why)) return fail(SPCONV_ERR_INVALID_ARG, why);
    if (n == 0) return SPCONV_OK;
    if (n > (int64_t(1) << 28)) return fail(SPCONV_ERR_INVALID_ARG, "8 n must stay below 2^31");
    if (!coords_out || !aligned16(coords_out))
        return fail(SPCONV_ERR_INVALID_ARG, "coords_out must be a 16-byte aligned device pointer");
    int64_t row_bytes = 0;
    if (x || x_out) {
        const spconv_status_t s = rows_arg_check(dtype, channels, x, x_out);
        if (s != SPCONV_OK) return s;
        row_bytes = (int64_t)channels * (dtype == SPCONV_BF16 ? 2 : 4);
    }
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int dev = 0;
    BuildAlloc al;
    al.stream = stream;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = device_pool(dev, &al.pool);
    auto* err = e == cudaSuccess ? al.temp<unsigned int>(1) : nullptr;
    if (e == cudaSuccess) e = al.err;
    unsigned int host_err = 0;
    if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(unsigned int), stream);
    if (e == cudaSuccess) e = spconv::launch_subdivide(coords, n, extent, row_bytes, x, coords_out, x_out, err, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_err, err, 4, cudaMemcpyDeviceToHost, stream);
    al.release_scratch();
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail_cuda(e, "spconv_subdivide");
    if (host_err & spconv::kErrCoordRange)
        return fail(SPCONV_ERR_COORD_RANGE, "a coordinate is outside [0, extent) or a batch index outside [0, 65535]");
    return SPCONV_OK;
}

}  // extern "C"
