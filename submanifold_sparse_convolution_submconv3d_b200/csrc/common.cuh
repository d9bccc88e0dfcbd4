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
};

// Device-side error bits written by forward kernels into the map's error word.
enum : unsigned int {
    kFwdErrTimeout = 1u,
};

struct BuildFlags {
    unsigned int err;
    unsigned int pad;
    unsigned long long pairs;  // (voxel, offset) pairs with an active neighbour, centre included
};

// Offset order used everywhere: k = (dx+1)*9 + (dy+1)*3 + (dz+1).
constexpr int kVol3 = 27;
constexpr int kCentre = 13;

// Tile metadata (built with the map, kernel size 3): the rows are cut into tiles
// of `tile_rows` consecutive rows (at most kTileRows, chosen per map by
// choose_tile_rows); for every tile and every non-centre offset the
// tile rows with an active neighbour there are listed, split into three classes
// by row % 3 and sorted by row within a class.  "Units" are (offset, class)
// pairs in offset-major order, offsets 0..26 without the centre: unit
// u = 3 * ks + c with ks = k < 13 ? k : k - 1.
constexpr int kTileRows = 384;
constexpr int kTileClasses = 3;
constexpr int kTileUnits = (kVol3 - 1) * kTileClasses;  // 78
constexpr int kTileCountStride = 80;                    // int32 counts per tile (78 used), 320 bytes
constexpr int kTileEntryAlign = 8;                      // each tile's entries start on a multiple of 8

__host__ __device__ inline int64_t num_tiles(int64_t n, int tile_rows) { return (n + tile_rows - 1) / tile_rows; }

// Rows per tile for n voxels on num_sms SMs (one tile per SM at a time): the
// number of waves that kTileRows-row tiles need, then the smallest tile that
// still fits n into that many waves, so the last wave is not left mostly empty.
inline int choose_tile_rows(int64_t n, int num_sms) {
    if (n <= 0 || num_sms <= 0) return kTileRows;
    const int64_t per_wave = (int64_t)kTileRows * num_sms;
    const int64_t waves = (n + per_wave - 1) / per_wave;
    const int64_t rows = (n + waves * num_sms - 1) / (waves * num_sms);
    return (int)(rows < 32 ? (n < 32 ? n : 32) : rows);
}

// The map handle (defined here so the launchers can read it).
struct MapData {
    int64_t n = 0;
    int32_t kernel_size = 3;
    int32_t extent[3] = {0, 0, 0};
    int64_t pairs = 0;
    int32_t* nbr = nullptr;        // device [n, 27] (kernel size 3), else null
    // tile metadata (kernel size 3): counts [ntiles][kTileCountStride]; tile_off
    // [ntiles + 2]: each tile's first entry (multiples of kTileEntryAlign), then the
    // grand total at slot ntiles and the largest tile's count at slot ntiles + 1;
    // local rows and neighbour rows per entry
    int32_t* tile_counts = nullptr;
    int64_t* tile_off = nullptr;
    uint16_t* pair_r = nullptr;
    int32_t* pair_j = nullptr;
    int64_t tile_entries = 0;
    int64_t tile_max_entries = 0;  // entries of the fullest tile (a multiple of kTileEntryAlign)
    int32_t tile_rows = kTileRows;  // rows per tile (<= kTileRows), for the forward kernels too
    unsigned int* fwd_err = nullptr;  // device word: forward-kernel error bits
    int device = 0;
    int num_sms = 0;
};

// Sets the calling thread's message returned by spconv_last_error().
void set_last_error(const std::string& msg);

// Launchers (each returns cudaSuccess or the first CUDA error).
cudaError_t launch_build_map(const int32_t* coords, int64_t n, const int32_t extent[3], int32_t kernel_size,
                             unsigned long long* table, uint64_t slots, int32_t* nbr, BuildFlags* flags,
                             cudaStream_t stream);

// Tile metadata in two passes: counts + offsets (then the caller reads the total
// and allocates the entry arrays), then the entries.
cudaError_t launch_tile_count(const int32_t* nbr, int64_t n, int tile_rows, int32_t* tile_counts, int64_t* tile_off,
                              cudaStream_t stream);
cudaError_t launch_tile_fill(const int32_t* nbr, int64_t n, int tile_rows, const int32_t* tile_counts,
                             const int64_t* tile_off, uint16_t* pair_r, int32_t* pair_j, cudaStream_t stream);

cudaError_t launch_forward_simt(const MapData& m, spconv_dtype_t dtype, const void* x, int cin, const void* w,
                                const void* bias, void* out, int cout, cudaStream_t stream);

// Returns SPCONV_OK, SPCONV_ERR_UNSUPPORTED (shape not handled) or SPCONV_ERR_CUDA.
spconv_status_t launch_forward_tcgen05(const MapData& m, const void* x, int cin, const void* w,
                                       const void* bias, void* out, int cout, cudaStream_t stream,
                                       cudaError_t* cuda_err);

}  // namespace spconv
