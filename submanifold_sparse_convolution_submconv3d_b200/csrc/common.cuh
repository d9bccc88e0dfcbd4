// Shared definitions of the SubMConv3d CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <string>

#include "spconv.h"

namespace spconv {

// Device-side error bits written by the build kernels (BuildFlags::err).
enum : unsigned int {
    kErrCoordRange = 1u,
    kErrDuplicate = 2u,
    kErrTableFull = 4u,
    kErrInternal = 8u,  // a bound the metadata relies on did not hold (not expected)
};

// Device-side error bits written by forward kernels into the map's error word.
enum : unsigned int {
    kFwdErrTimeout = 1u,
};

struct BuildFlags {
    unsigned int err;
    unsigned int pad;
    unsigned long long pairs;      // (voxel, offset) pairs with an active neighbour, centre included
    unsigned long long spans;      // window-kernel spans over all tiles
    unsigned long long span_cols;  // columns those spans cover
    unsigned long long max_tile_cols;  // longest per-tile index stream (columns of all its jobs)
};

// Offset order used everywhere: k = (dx+1)*9 + (dy+1)*3 + (dz+1).
constexpr int kVol3 = 27;
constexpr int kCentre = 13;

// Window-kernel metadata (kernel size 3).  The rows are reordered by their
// neighbour pattern: the 26 non-centre hit bits of a row form a mask, and the rows
// are sorted (stably) by the rank of that mask in the reflected Gray-code order,
// so rows with similar patterns sit next to each other and each offset's hits
// bunch into runs.  The sorted rows are cut into tiles of win_rows rows (a
// multiple of kWinCols, at most kWinMaxRows) and each tile into windows of
// kWinCols rows.  For every tile and non-centre offset, the windows holding a hit
// are covered by spans of consecutive windows (chosen by a cost model of the MMA,
// see map_window.cu); one span is one MMA of N = 16 * windows columns.  A tile's
// job list is its centre job (every row, N = win_rows) followed by its spans.
constexpr int kWinCols = 16;                 // rows per window (MMA N granule)
constexpr int kWinMaxRows = 256;             // rows per tile at most (one TMEM accumulator)
constexpr int kWinMaxSpans = 8;              // spans per (tile, offset) at most: kWinMaxRows / kWinCols / 2
// A tile's record (uint32 words): [0] job count J, [1] index-stream entries,
// [2], [3] index-stream start (low, high word), then J job words (the centre job
// first), padded to kWinJobStride words (a multiple of 4, so records stay 16-byte
// aligned for bulk copies).
constexpr int kWinRecHeader = 4;
constexpr int kWinJobStride = 216;           // header + centre job + <= 26 * 8 spans, padding
// Job word: offset k in bits 0-4, first window in bits 8-12, window count in bits 16-20.
__host__ __device__ inline uint32_t win_job(int k, int w0, int nw) {
    return (uint32_t)k | ((uint32_t)w0 << 8) | ((uint32_t)nw << 16);
}
__host__ __device__ inline int win_job_k(uint32_t j) { return (int)(j & 31u); }
__host__ __device__ inline int win_job_w0(uint32_t j) { return (int)((j >> 8) & 31u); }
__host__ __device__ inline int win_job_nw(uint32_t j) { return (int)((j >> 16) & 31u); }

// Window-tile height for n rows on num_sms SMs.  Measured on B200 (128^3 random,
// 256^3 and 512^3 shells, 4 x 64^3 shells; 64-256-row tiles): 192 rows is the
// fastest height for 32- and 64-channel chunks, 128 rows for 128-channel chunks,
// whose 16 KB gather units make the B ring shallow (so the short-tiles option,
// for maps whose layers take 128 or more input channels, picks 128).  A set too
// small to give every SM a 192-row tile takes the multiple of kWinCols in
// [128, 192] that minimises the rows of the busiest SM (ties: the taller tile).
constexpr int kTileRowsDefault = 192;
constexpr int kTileRowsShort = 128;
inline int choose_win_rows(int64_t n, int num_sms, bool short_tiles) {
    if (short_tiles) return kTileRowsShort;
    if (n <= 0 || num_sms <= 0 || n >= (int64_t)num_sms * kTileRowsDefault) return kTileRowsDefault;
    int best = kTileRowsDefault;
    int64_t best_load = -1;
    for (int r = kTileRowsDefault; r >= kTileRowsShort; r -= kWinCols) {
        const int64_t tiles = (n + r - 1) / r;
        const int64_t load = (tiles + num_sms - 1) / num_sms * r;
        if (best_load < 0 || load < best_load) {
            best_load = load;
            best = r;
        }
    }
    return best;
}

// Fused epilogue of a forward: y = act(conv + bias) (+ residual), stored; per
// channel sums of the stored value and its square into stats[0..cout) and
// stats[cout..2 cout) when stats is set.
struct Epilogue {
    int act = SPCONV_ACT_NONE;
    const void* residual = nullptr;
    float* stats = nullptr;
};

__device__ __forceinline__ float epi_act(int act, float y) {
    if (act == SPCONV_ACT_RELU) return fmaxf(y, 0.0f);
    if (act == SPCONV_ACT_SILU) return y / (1.0f + expf(-y));
    if (act == SPCONV_ACT_GELU) return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
    return y;
}

// The map handle (defined here so the launchers can read it).
struct MapData {
    int64_t n = 0;
    int32_t kernel_size = 3;
    uint32_t flags = 0;            // spconv_map_flags_t bits the map was built with
    int32_t extent[3] = {0, 0, 0};
    int64_t pairs = 0;
    int32_t* nbr = nullptr;        // device [n, 27] (kernel size 3), else null
    // window-kernel metadata (kernel size 3): perm [n] (sorted position -> row);
    // nbr_t [27][npad], the neighbour row of sorted row r at offset k or -1 (rows
    // r >= n are padding, all -1); win_jobs [win_tiles][kWinJobStride]
    int32_t* perm = nullptr;
    int32_t* nbr_t = nullptr;
    uint32_t* win_jobs = nullptr;
    int64_t npad = 0;
    int64_t win_tiles = 0;
    int32_t win_rows = kWinMaxRows;
    // per-tile index streams: the source rows of every job of the tile, job after
    // job; tile t's stream is idx_stream[idx_off[t] .. idx_off[t + 1])
    int32_t* idx_stream = nullptr;
    int64_t* idx_off = nullptr;
    int64_t max_tile_cols = 0;
    // work counters of the forward's tile scheduler: launches take the slots in
    // turn; the build zeroes them and each launch leaves its slot at zero
    uint32_t* sched = nullptr;
    int32_t* win_order = nullptr;  // [win_tiles] tiles in claim order (most expensive first)
    int64_t win_spans = 0;         // spans over all tiles (MMA jobs besides the centre)
    int64_t win_span_cols = 0;     // columns those spans cover
    unsigned int* fwd_err = nullptr;  // device word: forward-kernel error bits
    int device = 0;
    int num_sms = 0;
};

constexpr int kSchedSlots = 64;

// Sets the calling thread's message returned by spconv_last_error().
void set_last_error(const std::string& msg);

// Options of the map build.  flip: gather p - d_k instead of p + d_k.  sorted:
// build the dictionary by radix-sorting the packed keys (skeys[0..1], svals[0..1]:
// n elements each; hist: radix_hist_words(n) words) and probe it by binary search
// instead of the hash table (table and slots unused).
struct MapBuildOpts {
    bool flip = false;
    bool sorted = false;
    uint64_t* skeys[2] = {nullptr, nullptr};
    int32_t* svals[2] = {nullptr, nullptr};
    uint32_t* hist = nullptr;
};

// Key bits of the sorted dictionary for an extent: 16 batch bits plus, per axis,
// the bits of extent - 1.
int sorted_key_bits(const int32_t extent[3]);

// Launchers (each returns cudaSuccess or the first CUDA error).
// Pack + validate + build the dictionary, then (kernel size 3) probe into the
// dense map `nbr` and, when `keys` is not null, the rows' sort keys (Gray rank of
// the neighbour mask).
cudaError_t launch_build_map(const int32_t* coords, int64_t n, const int32_t extent[3], int32_t kernel_size,
                             unsigned long long* table, uint64_t slots, int32_t* nbr, uint32_t* keys,
                             BuildFlags* flags, cudaStream_t stream, const MapBuildOpts& opts = MapBuildOpts());

// Stable radix sort of (key, value) pairs by the low key_bits bits: keys[0] holds
// the input keys and vals_in the input values (null: the element indices);
// keys[1], vals[0] and vals[1] are buffers of n elements; hist holds
// radix_hist_words(n) words.  The sorted pairs end in keys[*which], vals[*which].
int64_t radix_hist_words(int64_t n);
cudaError_t radix_sort_pairs(uint32_t* keys[2], const int32_t* vals_in, int32_t* vals[2], int64_t n, int key_bits,
                             uint32_t* hist, int* which, cudaStream_t stream);
cudaError_t radix_sort_pairs64(uint64_t* keys[2], const int32_t* vals_in, int32_t* vals[2], int64_t n, int key_bits,
                               uint32_t* hist, int* which, cudaStream_t stream);

// Window-kernel metadata from the dense map and the sorted rows.
cudaError_t launch_win_meta(const int32_t* nbr, const int32_t* sorted_rows, int64_t n, int rows, int64_t tiles,
                            int64_t npad, int32_t* perm, int32_t* nbr_t, uint32_t* jobs, int64_t* idx_off,
                            int32_t* idx_stream, BuildFlags* flags, cudaStream_t stream);

// Sort keys of the tile claim order (ascending key = descending estimated cost).
cudaError_t launch_win_cost(const uint32_t* jobs, int64_t tiles, uint32_t* keys, cudaStream_t stream);

cudaError_t launch_forward_simt(const MapData& m, spconv_dtype_t dtype, const void* x, int cin, const void* w,
                                const void* bias, void* out, int cout, const Epilogue& epi, cudaStream_t stream);

// Test hook of the tensor-core forward: force the weight-ring slots and B-ring
// units of later launches (0, 0: automatic).
void set_forced_ring_depths(int sa, int ub);

// Kernel size 1 as a weight-stationary tcgen05 GEMM (forward_gemm1.cu): bf16,
// cin % 64 == 0 with the weight slice and two x stages in shared memory (cin <=
// 704 when cout % 128 == 0, else 1472), cout % 64 == 0, n >= 128.  Returns SPCONV_OK,
// SPCONV_ERR_UNSUPPORTED (shape not handled) or SPCONV_ERR_CUDA.
spconv_status_t launch_forward_gemm1(const MapData& m, const void* x, int cin, const void* w, const void* bias,
                                     void* out, int cout, const Epilogue& epi, cudaStream_t stream,
                                     cudaError_t* cuda_err);

// Test hook of the kernel-size-1 GEMM: x stages of later launches (0: as many as fit).
void set_forced_gemm1_stages(int stages);

// Returns SPCONV_OK, SPCONV_ERR_UNSUPPORTED (shape not handled) or SPCONV_ERR_CUDA.
spconv_status_t launch_forward_tcgen05(const MapData& m, const void* x, int cin, const void* w,
                                       const void* bias, void* out, int cout, const Epilogue& epi,
                                       cudaStream_t stream, cudaError_t* cuda_err);

}  // namespace spconv
