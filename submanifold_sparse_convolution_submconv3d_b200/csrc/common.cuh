// Shared definitions of the SubMConv3d CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

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

// The map handle (defined here so the launchers can read it).
struct MapData {
    int64_t n = 0;
    int32_t kernel_size = 3;
    int32_t extent[3] = {0, 0, 0};
    int64_t pairs = 0;
    int32_t* nbr = nullptr;        // device [n, 27] (kernel size 3), else null
    unsigned int* fwd_err = nullptr;  // device word: forward-kernel error bits
    int device = 0;
    int num_sms = 0;
};

// Launchers (each returns cudaSuccess or the first CUDA error).
cudaError_t launch_build_map(const int32_t* coords, int64_t n, const int32_t extent[3], int32_t kernel_size,
                             unsigned long long* table, uint64_t slots, int32_t* nbr, BuildFlags* flags,
                             cudaStream_t stream);

cudaError_t launch_forward_simt(const MapData& m, spconv_dtype_t dtype, const void* x, int cin, const void* w,
                                const void* bias, void* out, int cout, cudaStream_t stream);

// Returns SPCONV_OK, SPCONV_ERR_UNSUPPORTED (shape not handled) or SPCONV_ERR_CUDA.
spconv_status_t launch_forward_tcgen05(const MapData& m, const void* x, int cin, const void* w,
                                       const void* bias, void* out, int cout, cudaStream_t stream,
                                       cudaError_t* cuda_err);

}  // namespace spconv
