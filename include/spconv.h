/*
 * spconv.h -- C ABI of the B200 (sm_100a) submanifold sparse 3-D convolution
 * library (SubMConv3d, kernel size 3 or 1, stride 1).
 *
 * The operation (lato.2_mrp_mlx README, sections "The scope, once measured",
 * "Status" and "Correctness"; pixal3d_mrp_mlx README, "Status", for the weight
 * layout):
 *
 *   out[i] = bias + sum over d in {-1,0,1}^3 with p_i + d active of
 *            W[k(d)]^T x[index of p_i + d]
 *
 * Outputs exist only at the input's active voxels (stride 1, no padding), the
 * neighbour is gathered at p + d (cross-correlation), a neighbour must share the
 * batch index, and neighbours outside [0, extent) are holes.  The offset order
 * is k(d) = (dx+1)*9 + (dy+1)*3 + (dz+1), dx slowest (x, y, z = coordinate
 * columns 1, 2, 3); the centre offset is k = 13.
 *
 * The neighbour map is built once per coordinate set and cached in a handle,
 * as the pages cache their prepared device index (lato.2_mrp_mlx README, "Fleet
 * benchmark"); the map build is the step the same section names as dominant
 * whenever coordinates change.  The trellis-mac article (section on sparse 3D
 * convolution, gather-scatter) builds a hash map of active voxel coordinates
 * first and probes it per kernel offset; the build here does the same on the GPU.
 *
 * Conventions for every call:
 *   - Pointers documented as "device" must point to memory of the current CUDA
 *     device, 16-byte aligned.  Pointers documented as "host" are host memory.
 *     The library checks null pointers, alignment and the documented sizes, but
 *     it cannot tell host memory from device memory or see a buffer's length:
 *     a host pointer, or a device buffer shorter than documented, where a device
 *     buffer is required is undefined behaviour.  (The Python binding checks
 *     devices and shapes before it calls in.)
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).
 *   - The caller owns every buffer it passes; the library keeps no pointer to a
 *     caller buffer after a call returns.
 *   - Errors are returned as spconv_status_t; nothing aborts or throws across
 *     the ABI.  spconv_last_error() gives a message for the calling thread's
 *     most recent failure.
 */
#ifndef SPCONV_B200_H
#define SPCONV_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define SPCONV_API __attribute__((visibility("default")))
#else
#define SPCONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct spconv_map_s* spconv_map_t; /* opaque, owned by the library */

typedef enum {
    SPCONV_OK = 0,
    SPCONV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad alignment, bad extent */
    SPCONV_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. bf16 with C % 16 != 0) */
    SPCONV_ERR_COORD_RANGE = 3,  /* a coordinate outside [0, extent) or batch outside [0, 65535] */
    SPCONV_ERR_DUPLICATE = 4,    /* the same (b, x, y, z) appears twice */
    SPCONV_ERR_TABLE_FULL = 5,   /* the hash table ran out of slots */
    SPCONV_ERR_OOM = 6,          /* a device allocation failed */
    SPCONV_ERR_CUDA = 7,         /* a CUDA runtime call failed */
    SPCONV_ERR_TIMEOUT = 8       /* a bounded device-side wait gave up */
} spconv_status_t;

typedef enum { SPCONV_F32 = 0, SPCONV_BF16 = 1 } spconv_dtype_t;

/*
 * Build the neighbour map of a coordinate set.
 *
 *   coords       device int32 [n, 4], row-major, columns (b, x, y, z).
 *   n            number of active voxels, 0 <= n < 2^31.  n = 0 gives an empty map.
 *   extent       host int32 [3] = (X, Y, Z), each in [1, 65535].
 *   kernel_size  3 (27 offsets) or 1 (the map is the identity and is not stored).
 *   stream       stream on which the build runs.
 *   out_map      receives the handle on success; untouched on failure.
 *
 * Device work: pack (b, x, y, z) into a 64-bit key and validate it; insert the
 * keys into an open-addressing hash table (linear probing, 64-bit CAS, load
 * factor <= 1/2; spconv_build_map_ex can build radix-sorted keys instead); probe
 * the 26 neighbours of every voxel (the first slots of three offsets loaded
 * together) and write the dense map nbr[i*27 + k] = row of p_i + d_k, or -1.  For kernel size 3 it then prepares
 * the tensor-core forward's metadata: the rows sorted (stably, on the GPU) by the
 * Gray-code rank of their 26-bit neighbour mask, the neighbour table in that
 * order, and per tile of sorted rows the MMA jobs (see spconv_map_stats).
 * Memory: every buffer comes from a stream-ordered memory pool the library keeps
 * per device, allocated on `stream`; the hash table and sort scratch go back to
 * the pool on `stream` before the call returns.  No cudaMalloc or cudaFree is
 * called, and the device is not synchronised.
 * Synchronisation: the call synchronises `stream` once, at the end, to read the
 * device error flags, and returns only a valid map.
 * Errors: SPCONV_ERR_COORD_RANGE, SPCONV_ERR_DUPLICATE, SPCONV_ERR_TABLE_FULL,
 * SPCONV_ERR_INVALID_ARG, SPCONV_ERR_OOM, SPCONV_ERR_CUDA.
 * The map may be used on any stream of the same device after the call returns.
 */
SPCONV_API spconv_status_t spconv_build_map(const int32_t* coords, int64_t n, const int32_t* extent,
                                 int32_t kernel_size, void* stream, spconv_map_t* out_map);

/*
 * Options of spconv_build_map_ex (bits of `flags`).
 *
 *   SPCONV_MAP_FLIP_KERNEL  gather x at p - d_k instead of p + d_k: the kernel
 *                           is mirrored (a true convolution rather than a
 *                           cross-correlation).  The lato.2_mrp_mlx README
 *                           ("Correctness") leaves open which of the two the
 *                           upstream library computes and builds the mirrored
 *                           one behind its --flip-kernel switch.  The map is the
 *                           default map with offsets k and 26 - k exchanged.
 *   SPCONV_MAP_SORTED_KEYS  build the coordinate dictionary by radix-sorting the
 *                           packed keys and find every neighbour by binary search
 *                           -- the sorted-key index map that the lato.2_mrp_mlx
 *                           README's table of upstream equivalents gives for its
 *                           port -- instead of the hash table.  Same map, bit for bit.
 *                           Needs 16 + sum over axes of ceil(log2(extent)) <= 62
 *                           (SPCONV_ERR_UNSUPPORTED otherwise); never reports
 *                           SPCONV_ERR_TABLE_FULL.
 *   SPCONV_MAP_HASH_TABLE   build with the hash table (the default).
 *   SPCONV_MAP_SHORT_TILES  cut the sorted rows into 128-row tiles instead of 192:
 *                           faster for layers with 128 or more input channels
 *                           (their 16 KB gather units leave room for fewer jobs
 *                           in flight), slower for narrower ones.  Same results.
 * With neither dictionary flag the library builds the hash table.  Both flags
 * together: SPCONV_ERR_INVALID_ARG.
 */
typedef enum {
    SPCONV_MAP_DEFAULT = 0,
    SPCONV_MAP_FLIP_KERNEL = 1,
    SPCONV_MAP_SORTED_KEYS = 2,
    SPCONV_MAP_HASH_TABLE = 4,
    SPCONV_MAP_SHORT_TILES = 8
} spconv_map_flags_t;

/*
 * spconv_build_map with options: `flags` is a bitwise OR of spconv_map_flags_t
 * values (an unknown bit: SPCONV_ERR_INVALID_ARG).  Everything else, including
 * memory, synchronisation and errors, is as spconv_build_map, which is this call
 * with flags = SPCONV_MAP_DEFAULT.  The forward runs unchanged on either map.
 */
SPCONV_API spconv_status_t spconv_build_map_ex(const int32_t* coords, int64_t n, const int32_t* extent,
                                               int32_t kernel_size, uint32_t flags, void* stream,
                                               spconv_map_t* out_map);

/*
 * Run one SubMConv3d layer over a map.
 *
 *   map     handle from spconv_build_map.
 *   dtype   element type shared by x, w, bias and out (SPCONV_F32 or SPCONV_BF16).
 *   x       device [n, cin] row-major, row i = voxel i of the map's coordinates.
 *   cin     input channels (bf16: a multiple of 16).
 *   w       device [K^3, cin, cout] row-major (K^3 = 27 or 1), offset order above.
 *   bias    device [cout] or NULL (no bias).
 *   out     device [n, cout] row-major; must not overlap x.  Each row is written once.
 *   cout    output channels (bf16: a multiple of 16).
 *   stream  stream on which the layer runs.
 *
 * Accumulation is fp32 in every mode; the bf16 result is rounded to nearest even.
 * bf16 with cout a multiple of 64 runs on the tensor cores (tcgen05): a map of
 * kernel size 1 with cin a multiple of 64 (cin <= 704 when cout % 128 == 0, else
 * cin <= 1472) and n >= 128 on a weight-stationary GEMM, every other such layer
 * on the window kernel; fp32, and bf16 with other channel counts, on a CUDA-core
 * kernel.  The choice depends on dtype, the kernel size, n and the channel
 * counts alone; spconv_map_launch_counts reports which kernel ran.
 * The layer runs on the current CUDA device, which must be the device the map
 * was built on (otherwise SPCONV_ERR_INVALID_ARG).
 * The call only validates on the host and launches; it never synchronises.
 * Errors: SPCONV_ERR_INVALID_ARG, SPCONV_ERR_UNSUPPORTED, SPCONV_ERR_CUDA.  A
 * device-side wait that gives up is recorded in the map and reported by
 * spconv_map_check().
 */
SPCONV_API spconv_status_t spconv_subm_forward(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                    const void* w, const void* bias, void* out, int32_t cout,
                                    void* stream);

/* Release a map.  The call synchronises the map's device (kernels on any stream
 * may still read the map), then returns the map's memory to the library's pool.
 * NULL is accepted and ignored. */
SPCONV_API spconv_status_t spconv_free(spconv_map_t map);

/*
 * Introspection of a map (for tests and the benchmark).
 *   n            receives the voxel count (may be NULL).
 *   kernel_size  receives 3 or 1 (may be NULL).
 *   pairs        receives the number of (voxel, offset) pairs with an active
 *                neighbour, the centre included (n for kernel size 1) (may be NULL).
 *   nbr_dev      receives the device pointer of the dense int32 [n, 27] map, or
 *                NULL for kernel size 1 or n = 0 (may be NULL).  The library owns it.
 */
SPCONV_API spconv_status_t spconv_map_info(spconv_map_t map, int64_t* n, int32_t* kernel_size, int64_t* pairs,
                                const int32_t** nbr_dev);

/*
 * Rows per tile (a multiple of 16, at most 256) that the tensor-core forward uses
 * with this map: 192, or 128 with SPCONV_MAP_SHORT_TILES; a set too small to give
 * every SM a 192-row tile takes the height in [128, 192] that evens out the rows
 * of the busiest SM; spconv_debug_set_tile_rows forces it.  For reports and tests; no device work.
 * A null `map` or `rows` returns SPCONV_ERR_INVALID_ARG.
 */
SPCONV_API spconv_status_t spconv_map_tile_rows(spconv_map_t map, int32_t* rows);

/*
 * The tensor-core forward's metadata of a kernel-size-3 map (for reports and
 * tests; no device work).  The rows are sorted by the Gray-code rank of their
 * neighbour mask (bit 25 - ks for offset k, ks = k < 13 ? k : k - 1) and cut into
 * `tiles` tiles of `rows_per_tile` sorted rows; a tile's rows are cut into windows
 * of 16.  For every tile and non-centre offset, the windows holding a neighbour
 * are covered by spans of consecutive windows; each span is one tensor-core job
 * of 16 * windows columns (holes inside it are multiplied as zero rows).
 *   tiles, rows_per_tile  tiling of the sorted rows (0 tiles for n = 0)
 *   spans, span_cols      spans over all tiles and the columns they cover
 *   perm_dev              device int32 [n]: the row at each sorted position
 *   nbr_t_dev             device int32 [27][tiles * rows_per_tile]: the neighbour
 *                         row of sorted row r at offset k, -1 for none and for
 *                         padding rows r >= n
 *   jobs_dev              device uint32 [tiles][job_stride]: word 0 = job count J,
 *                         word 1 = length of the tile's index stream (the source
 *                         rows of all its jobs, job after job), words 2, 3 = its
 *                         start (low, high), words 4 .. 3 + J = jobs, each k |
 *                         first window << 8 | windows << 16; the first job is the
 *                         centre (k = 13, all windows), the spans of each offset
 *                         follow in increasing order
 *   order_dev             device int32 [tiles]: the order in which the forward's
 *                         CTAs claim the tiles, by descending estimated cost
 *                         (4 * J + stream length / 16) / 4, integer divisions
 *                         (stable: ties by tile index)
 * Pointers are NULL for kernel size 1 and n = 0.  The library owns them.
 * A null `map` or `stats` returns SPCONV_ERR_INVALID_ARG.
 */
typedef struct {
    int64_t tiles;
    int32_t rows_per_tile;
    int32_t job_stride;
    int64_t spans;
    int64_t span_cols;
    const int32_t* perm_dev;
    const int32_t* nbr_t_dev;
    const uint32_t* jobs_dev;
    const int32_t* order_dev;
} spconv_map_stats_t;
SPCONV_API spconv_status_t spconv_map_stats(spconv_map_t map, spconv_map_stats_t* stats);

/*
 * Synchronise `stream` and report (then clear) any device-side wait of a forward
 * kernel on this map that gave up: SPCONV_OK or SPCONV_ERR_TIMEOUT.  After a
 * timeout it also resets the map's tile-scheduler counters; call it before the
 * map's next forward.
 */
SPCONV_API spconv_status_t spconv_map_check(spconv_map_t map, void* stream);

/* Message for the calling thread's most recent failure ("" if none). */
SPCONV_API const char* spconv_last_error(void);

/*
 * Forward with an explicit kernel family, for cross-checks:
 *   SPCONV_ALGO_AUTO     what spconv_subm_forward uses: the tcgen05 kernels for
 *                        bf16 when cout % 64 == 0 (the GEMM or the window kernel,
 *                        as described there), the CUDA-core kernel otherwise.
 *   SPCONV_ALGO_SIMT     CUDA-core FMA kernel, any channel count, fp32 or bf16.
 *   SPCONV_ALGO_TCGEN05  the tcgen05 tensor-core kernels (bf16, cin % 16 == 0,
 *                        cout % 64 == 0; SPCONV_ERR_UNSUPPORTED otherwise): the
 *                        same GEMM-or-window choice as AUTO.
 * Same arguments, ownership and errors as spconv_subm_forward.
 */
typedef enum { SPCONV_ALGO_AUTO = 0, SPCONV_ALGO_SIMT = 1, SPCONV_ALGO_TCGEN05 = 2 } spconv_algo_t;
SPCONV_API spconv_status_t spconv_subm_forward_algo(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                         const void* w, const void* bias, void* out, int32_t cout,
                                         spconv_algo_t algo, void* stream);

/*
 * Fused decoder epilogue of a forward (spconv_subm_forward_ex).  The
 * pixal3d_mrp_mlx README ("Correction to the earlier scope") lists the ConvNeXt
 * and ResBlock decoder blocks around the convolution; the lato.2_mrp_mlx README
 * ("Status") lists the activations, norms and SparseResBlock of the shared core.
 * The store of each output element then computes, in fp32,
 *
 *   y = act(conv + bias) (+ residual),  out = y rounded to the dtype,
 *
 * and, when `stats` is given, adds out and out^2 into per-channel sums over all
 * rows (what a following LayerNorm / GroupNorm reads).
 *
 *   act       SPCONV_ACT_NONE, _RELU (max(y, 0)), _SILU (y / (1 + exp(-y))) or
 *             _GELU (0.5 y (1 + erf(y / sqrt 2)), the exact form).
 *   residual  device [n, cout] of the forward's dtype, 16-byte aligned, or NULL.
 *             It may be `out` itself (each element is read before it is
 *             written); it must not otherwise overlap out, and must not overlap x.
 *   stats     device fp32 [2, cout], 16-byte aligned, or NULL: row 0 receives the
 *             per-channel sum of the stored output, row 1 the sum of squares.  The
 *             call zeroes it on `stream` first; the sums are accumulated with fp32
 *             atomics, so their last bits depend on the order of the additions.
 */
typedef enum { SPCONV_ACT_NONE = 0, SPCONV_ACT_RELU = 1, SPCONV_ACT_SILU = 2, SPCONV_ACT_GELU = 3 } spconv_act_t;
typedef struct {
    spconv_act_t act;
    const void* residual;
    float* stats;
} spconv_epilogue_t;

/*
 * spconv_subm_forward_algo with a fused epilogue.  `epi` may be NULL (no
 * epilogue).  Same arguments, ownership, synchronisation (none) and errors as
 * spconv_subm_forward_algo, plus SPCONV_ERR_INVALID_ARG for an unknown act, a
 * misaligned residual or stats, or a residual overlapping x or partly overlapping
 * out.  Both kernel families apply the epilogue.
 */
SPCONV_API spconv_status_t spconv_subm_forward_ex(spconv_map_t map, spconv_dtype_t dtype, const void* x, int32_t cin,
                                                  const void* w, const void* bias, void* out, int32_t cout,
                                                  const spconv_epilogue_t* epi, spconv_algo_t algo, void* stream);

/*
 * Kernel families a forward can run on, for spconv_map_launch_counts.
 */
typedef enum {
    SPCONV_KERNEL_SIMT = 0,     /* CUDA-core FMA kernel: fp32, and bf16 shapes no tensor-core kernel takes */
    SPCONV_KERNEL_TCGEN05 = 1,  /* tcgen05 tensor-core window kernel (gathered rows) */
    SPCONV_KERNEL_TCGEN05_GEMM = 2, /* tcgen05 weight-stationary GEMM: kernel size 1, cin % 64 == 0, n >= 128 */
    SPCONV_KERNEL_KINDS = 3
} spconv_kernel_t;

/*
 * Forward launches made on this map since it was built, per kernel family:
 * counts[k] receives the launches of family k for k < min(ncounts,
 * SPCONV_KERNEL_KINDS); entries beyond SPCONV_KERNEL_KINDS are set to 0.  Lets a
 * caller (and the tests) see which kernel SPCONV_ALGO_AUTO chose.  Host-side
 * counters only: no device work.  A null map or counts, or ncounts < 1:
 * SPCONV_ERR_INVALID_ARG.
 */
SPCONV_API spconv_status_t spconv_map_launch_counts(spconv_map_t map, int64_t* counts, int32_t ncounts);

/*
 * Test hook: force the hash-table slot count of later builds in this process
 * (0 restores the automatic choice, a power of two >= 2n).  Lets a test reach
 * SPCONV_ERR_TABLE_FULL with a small table.  `slots` must be 0 or a power of two.
 */
SPCONV_API spconv_status_t spconv_debug_set_table_slots(int64_t slots);

/*
 * Test hook: force the tile height (sorted rows per tile, a multiple of 16 in
 * [16, 256]) of later builds in this process; 0 restores the automatic choice.
 * Lets tests run small inputs through full-height tiles and many short tiles.
 * Other values: SPCONV_ERR_INVALID_ARG.
 */
SPCONV_API spconv_status_t spconv_debug_set_tile_rows(int32_t rows);

/*
 * Test hook: force the tensor-core forward's ring depths for later launches in
 * this process: a_slots weight tiles in [2, 8] and b_units units of 64 gathered
 * rows in [4, 32]; (0, 0) restores the automatic choice.  A launch whose forced
 * depths do not fit shared memory returns SPCONV_ERR_UNSUPPORTED.  The
 * kernel-size-1 GEMM takes a_slots as its count of x stages (fewer if they do
 * not fit).  Lets tests drive shallow rings (frequent wrap-around) and the
 * benchmark sweep depths.
 * Other values: SPCONV_ERR_INVALID_ARG.
 */
SPCONV_API spconv_status_t spconv_debug_set_ring_depths(int32_t a_slots, int32_t b_units);

/*
 * Neighbour-map build that allocates no device memory.  The pages have no
 * counterpart: this is an interface for callers that cannot call cudaMalloc or
 * cudaFree -- code running while another component owns the device memory (a
 * framework's caching allocator, an arena reserved up front) and latency-critical
 * loops, since cudaFree synchronises the whole device and cudaMalloc can stall
 * other streams.
 *
 *   coords     device int32 [n, 4] (b, x, y, z), 16-byte aligned.
 *   n          0 <= n <= 524288 (larger sets: SPCONV_ERR_UNSUPPORTED; use spconv_build_map).
 *   extent     host int32 [3], each in [1, 65535].
 *   nbr_out    device int32 [n, 27], caller-owned: nbr_out[i*27 + k] = row of the
 *              active voxel at p_i + d_k, or -1 (same values as the map that
 *              spconv_build_map builds with kernel size 3).
 *   pairs_out  host; receives the number of entries >= 0 of nbr_out (may be NULL).
 *   stream     stream on which the build runs; the call synchronises it once.
 *
 * The hash table and error flags live in one static device array of 16 MiB plus
 * 256 bytes that every GPU loading this library holds until the process exits.
 * Every call looks up that array's device address with the calling thread's
 * current device (the lookup allocates nothing), so the entry point stays valid
 * after a device reset.  The first call on a device may load the library's
 * device code there.  Every call shares the array and clears it before use, so
 * calls that overlap on the GPU (on different streams or host threads) race and
 * must not be issued.  The call copies the error flags to host memory and
 * synchronises `stream` before it returns, so it must never be issued while
 * `stream` (or any stream it would join) is being captured into a CUDA graph.
 * Errors: as spconv_build_map, plus SPCONV_ERR_UNSUPPORTED above the size limit;
 * spconv_last_error() describes them.
 */
SPCONV_API spconv_status_t spconv_build_neighbor_map_noalloc(const int32_t* coords, int64_t n, const int32_t* extent,
                                                             int32_t* nbr_out, int64_t* pairs_out, void* stream);

/*
 * ---------------------------------------------------------------- resampling
 * The sparse ops that change the coordinate set around the convolution: the
 * lato.2_mrp_mlx README ("Status") lists SparseDownsample as max pooling with
 * the "amax" reduction; its table of upstream equivalents does upsampling with
 * SparseSubdivide, a x8 expansion of the coordinates; the pixal3d_mrp_mlx README
 * ("Scope, measured against the shared core") has SparseUpsample(2) as the
 * inverse of a downsample that reuses the downsample's pairing.  A convolution
 * on the new set needs a new neighbour map (spconv_build_map).
 */
typedef struct spconv_downsample_s* spconv_downsample_t; /* opaque, owned by the library */

/*
 * SparseDownsample(factor) coordinates.  Every voxel (b, x, y, z) falls in the
 * coarse voxel (b, x / factor, y / factor, z / factor) (integer division); the
 * coarse set is the set of those, in increasing lexicographic (b, x, y, z) order,
 * on the grid ceil(extent / factor).
 *
 *   coords   device int32 [n, 4] (b, x, y, z), 16-byte aligned; no duplicates
 *            needed for correctness (a repeated voxel just joins its block twice).
 *   n        0 <= n < 2^31.
 *   extent   host int32 [3], each in [1, 65535].
 *   factor   block edge, in [1, 65535] (the pages use 2).
 *   stream   stream on which the build runs; the call synchronises it once, at
 *            the end, to read the coarse count and the error flag.
 *   out      receives the handle on success; untouched on failure.
 *
 * Device work: pack each voxel's coarse key (bit fields sized by the coarse
 * extent), radix-sort (key, row) stably, number the runs of equal keys by a scan,
 * write the coarse coordinates, each run's start and each fine row's parent.
 * Memory comes from the library's stream-ordered pool, as for spconv_build_map;
 * spconv_downsample_free returns it.
 * Errors: SPCONV_ERR_INVALID_ARG, SPCONV_ERR_COORD_RANGE, SPCONV_ERR_OOM,
 * SPCONV_ERR_CUDA.
 */
SPCONV_API spconv_status_t spconv_downsample_build(const int32_t* coords, int64_t n, const int32_t* extent,
                                                   int32_t factor, void* stream, spconv_downsample_t* out);

/*
 * Introspection of a downsample (any pointer may be NULL):
 *   n_fine             input voxel count n
 *   n_coarse           coarse voxel count
 *   coarse_extent      host int32 [3]: ceil(extent / factor)
 *   coarse_coords_dev  device int32 [n_coarse, 4] (b, x, y, z), sorted, 16-byte
 *                      aligned: a valid `coords` argument for spconv_build_map
 *   parent_dev         device int32 [n]: coarse row of every input row
 * The library owns the buffers (NULL when n = 0).
 */
SPCONV_API spconv_status_t spconv_downsample_info(spconv_downsample_t ds, int64_t* n_fine, int64_t* n_coarse,
                                                  int32_t* coarse_extent, const int32_t** coarse_coords_dev,
                                                  const int32_t** parent_dev);

/*
 * Max pooling over a downsample: out[g, c] = max over input rows i with
 * parent[i] = g of x[i, c] ("amax").  Exact; where the maximum is a zero, +0
 * wins over -0 (the IEEE 754 total order).  NaN inputs give unspecified values.
 *
 *   x        device [n, channels] of dtype, row-major, 16-byte aligned.
 *   out      device [n_coarse, channels] of dtype, 16-byte aligned; must not
 *            overlap x.
 * Asynchronous on `stream` (no synchronisation).  The current device must be the
 * handle's.  Errors: SPCONV_ERR_INVALID_ARG, SPCONV_ERR_CUDA.
 */
SPCONV_API spconv_status_t spconv_downsample_amax(spconv_downsample_t ds, spconv_dtype_t dtype, const void* x,
                                                  int32_t channels, void* out, void* stream);

/*
 * SparseUpsample paired with a downsample: out[i, :] = x_coarse[parent[i], :],
 * back on the downsample's input voxels, in their input order.
 *
 *   x_coarse  device [n_coarse, channels] of dtype, 16-byte aligned.
 *   out       device [n, channels] of dtype, 16-byte aligned.
 * Asynchronous; same errors as spconv_downsample_amax.
 */
SPCONV_API spconv_status_t spconv_upsample(spconv_downsample_t ds, spconv_dtype_t dtype, const void* x_coarse,
                                           int32_t channels, void* out, void* stream);

/* Release a downsample (synchronises its device first, like spconv_free).  NULL
 * is accepted and ignored. */
SPCONV_API spconv_status_t spconv_downsample_free(spconv_downsample_t ds);

/*
 * SparseSubdivide: every voxel becomes its 8 children on the grid 2 * extent.
 * Output row 8 i + c, c = 4 ox + 2 oy + oz with ox, oy, oz in {0, 1}, is the
 * voxel (b, 2x + ox, 2y + oy, 2z + oz) and carries row i's features.
 *
 *   coords      device int32 [n, 4] (b, x, y, z), 16-byte aligned.
 *   n           0 <= n <= 2^28.
 *   extent      host int32 [3], each in [1, 32767] (the doubled grid must stay
 *               within 65535).
 *   dtype, x, channels   device features [n, channels], or x = NULL and
 *               x_out = NULL to expand the coordinates only.
 *   coords_out  device int32 [8n, 4], 16-byte aligned.
 *   x_out       device [8n, channels] of dtype, 16-byte aligned.
 *   stream      the call synchronises it once, to read the range check.
 * Errors: SPCONV_ERR_INVALID_ARG, SPCONV_ERR_COORD_RANGE (a coordinate outside
 * [0, extent); the outputs are then unspecified), SPCONV_ERR_OOM, SPCONV_ERR_CUDA.
 */
SPCONV_API spconv_status_t spconv_subdivide(const int32_t* coords, int64_t n, const int32_t* extent,
                                            spconv_dtype_t dtype, const void* x, int32_t channels,
                                            int32_t* coords_out, void* x_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPCONV_B200_H */
