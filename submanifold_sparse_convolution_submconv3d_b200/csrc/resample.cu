// Coordinate-changing neighbours of the convolution: SparseDownsample (max
// pooling over factor^3 blocks), its cache-paired inverse SparseUpsample, and
// SparseSubdivide (every voxel becomes its 8 children).
//
// The pages list these as the sparse ops around the convolution: the
// lato.2_mrp_mlx README ("Status") has SparseDownsample as max pooling with the
// "amax" reduction, not an average, and its table of upstream equivalents has
// upsampling done by SparseSubdivide, a x8 expansion of the coordinates; the
// pixal3d_mrp_mlx README ("Scope, measured against the shared core") has
// SparseUpsample(2) as the inverse of a downsample that reuses the downsample's
// cached pairing.  Each produces a new coordinate set, so a convolution after it
// needs a new neighbour map (the lato.2_mrp_mlx README, "Fleet benchmark": the
// map build matters whenever coordinates change).
//
// Downsample build: every voxel's coarse key (b, x / f, y / f, z / f), packed as
// in the sorted-key map build, is radix-sorted with its row; the first position
// of each run of equal keys starts a coarse voxel, numbered by a scan, so the
// coarse voxels come out in lexicographic (b, x, y, z) order.  The pooling then
// reads, per coarse voxel and 16-byte chunk of channels, the rows of its run.
#include "common.cuh"

namespace spconv {
namespace {

constexpr int kScanBlock = 1024;  // positions per block of the run-numbering scan

int bits_of(int extent) {
    int b = 0;
    while ((1 << b) < extent) ++b;
    return b;
}

struct CoarseBits {
    int bz, by, bx;
};

__device__ __forceinline__ unsigned long long coarse_key(CoarseBits kb, unsigned b, unsigned x, unsigned y, unsigned z) {
    return ((unsigned long long)b << (kb.bx + kb.by + kb.bz)) | ((unsigned long long)x << (kb.by + kb.bz)) |
           ((unsigned long long)y << kb.bz) | (unsigned long long)z;
}

__global__ void k_ds_pack(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez, int f, CoarseBits kb,
                          unsigned long long* __restrict__ keys, unsigned int* __restrict__ err) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int4 c = coords[i];
    if ((unsigned)c.x > 65535u || (unsigned)c.y >= (unsigned)ex || (unsigned)c.z >= (unsigned)ey ||
        (unsigned)c.w >= (unsigned)ez) {
        atomicOr(err, kErrCoordRange);
        keys[i] = 0;
        return;
    }
    keys[i] = coarse_key(kb, c.x, c.y / f, c.z / f, c.w / f);
}

__device__ __forceinline__ bool run_head(const unsigned long long* __restrict__ sk, int64_t s) {
    return s == 0 || sk[s] != sk[s - 1];
}

// Per block of kScanBlock sorted positions: how many runs start in it.
__global__ void __launch_bounds__(256) k_ds_count(const unsigned long long* __restrict__ sk, int64_t n,
                                                  uint32_t* __restrict__ counts) {
    const int64_t s0 = (int64_t)blockIdx.x * kScanBlock;
    uint32_t c = 0;
    for (int e = threadIdx.x; e < kScanBlock; e += blockDim.x) {
        const int64_t s = s0 + e;
        if (s < n && run_head(sk, s)) ++c;
    }
    for (int d = 16; d > 0; d >>= 1) c += __shfl_down_sync(0xffffffffu, c, d);
    __shared__ uint32_t part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
        counts[blockIdx.x] = t;
    }
}

// Exclusive scan of the block counts in place (one CTA); counts[blocks] receives
// the total, the number of coarse voxels.
__global__ void __launch_bounds__(1024) k_ds_scan(uint32_t* __restrict__ counts, int64_t blocks) {
    __shared__ uint32_t part[1024];
    const int64_t per = (blocks + blockDim.x - 1) / blockDim.x;
    const int64_t lo = threadIdx.x * per, hi = min(blocks, lo + per);
    uint32_t sum = 0;
    for (int64_t i = lo; i < hi; ++i) sum += counts[i];
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int d = 1; d < (int)blockDim.x; d <<= 1) {
        const uint32_t v = threadIdx.x >= (unsigned)d ? part[threadIdx.x - d] : 0u;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    uint32_t run = part[threadIdx.x] - sum;
    for (int64_t i = lo; i < hi; ++i) {
        const uint32_t v = counts[i];
        counts[i] = run;
        run += v;
    }
    if (threadIdx.x == blockDim.x - 1) counts[blocks] = part[threadIdx.x];
}

// Numbers the runs: position s with run index g writes parent[row] = g; a run's
// first position also writes the coarse voxel's coordinates and its run start.
__global__ void __launch_bounds__(kScanBlock) k_ds_emit(const unsigned long long* __restrict__ sk,
                                                        const int32_t* __restrict__ srows, int64_t n, CoarseBits kb,
                                                        const uint32_t* __restrict__ offs, int4* __restrict__ coarse,
                                                        int32_t* __restrict__ seg, int32_t* __restrict__ parent) {
    __shared__ uint32_t wsum[kScanBlock / 32];
    const int64_t s = (int64_t)blockIdx.x * kScanBlock + threadIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool valid = s < n;
    const uint32_t h = valid && run_head(sk, s) ? 1u : 0u;
    // inclusive scan of the head flags over the block
    uint32_t v = h;
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += t;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = wsum[lane];
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w += t;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    const uint32_t incl = v + (warp > 0 ? wsum[warp - 1] : 0u) + offs[blockIdx.x];
    if (!valid) return;
    const int32_t g = (int32_t)incl - 1;  // the run holding position s
    parent[srows[s]] = g;
    if (h) {
        const unsigned long long key = sk[s];
        const int z = (int)(key & ((1ull << kb.bz) - 1));
        const int y = (int)((key >> kb.bz) & ((1ull << kb.by) - 1));
        const int x = (int)((key >> (kb.by + kb.bz)) & ((1ull << kb.bx) - 1));
        const int b = (int)(key >> (kb.bx + kb.by + kb.bz));
        coarse[g] = make_int4(b, x, y, z);
        seg[g] = (int32_t)s;
    }
    if (s == n - 1) seg[g + 1] = (int32_t)n;
}

// Order-preserving integer image of a float's bits: larger values map to larger
// integers, and -0 maps below +0 (the IEEE 754 totalOrder on non-NaN values).
__device__ __forceinline__ uint32_t ord16(uint32_t u) { return (u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u); }
__device__ __forceinline__ uint32_t unord16(uint32_t o) { return (o & 0x8000u) ? (o & 0x7FFFu) : (~o & 0xFFFFu); }
__device__ __forceinline__ uint32_t ord32(uint32_t u) { return (u & 0x80000000u) ? ~u : (u | 0x80000000u); }
__device__ __forceinline__ uint32_t unord32(uint32_t o) { return (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o; }

// Max of one 32-bit word of a run, element-wise: two bf16 or one fp32.
template <bool kBf16>
__device__ __forceinline__ uint32_t word_ord(uint32_t w) {
    if constexpr (kBf16) return ord16(w & 0xFFFFu) | (ord16(w >> 16) << 16);
    else return ord32(w);
}
template <bool kBf16>
__device__ __forceinline__ uint32_t word_unord(uint32_t o) {
    if constexpr (kBf16) return unord16(o & 0xFFFFu) | (unord16(o >> 16) << 16);
    else return unord32(o);
}
template <bool kBf16>
__device__ __forceinline__ uint32_t word_max(uint32_t a, uint32_t b) {
    if constexpr (kBf16) {
        return max(a & 0xFFFFu, b & 0xFFFFu) | (max(a >> 16, b >> 16) << 16);
    } else {
        return max(a, b);
    }
}

// One thread per (coarse voxel, 16-byte chunk): the element-wise maximum over the
// run's rows, in the order image so every comparison is an integer one.
template <bool kBf16>
__global__ void k_ds_amax(const int32_t* __restrict__ seg, const int32_t* __restrict__ srows, int64_t ncoarse,
                          int chunks, const uint4* __restrict__ x, uint4* __restrict__ out) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= ncoarse * chunks) return;
    const int64_t g = t / chunks;
    const int q = (int)(t % chunks);
    const int32_t s0 = seg[g], s1 = seg[g + 1];
    uint4 m = make_uint4(0, 0, 0, 0);  // below every order image
    for (int32_t s = s0; s < s1; ++s) {
        const uint4 v = x[(int64_t)srows[s] * chunks + q];
        m.x = word_max<kBf16>(m.x, word_ord<kBf16>(v.x));
        m.y = word_max<kBf16>(m.y, word_ord<kBf16>(v.y));
        m.z = word_max<kBf16>(m.z, word_ord<kBf16>(v.z));
        m.w = word_max<kBf16>(m.w, word_ord<kBf16>(v.w));
    }
    out[t] = make_uint4(word_unord<kBf16>(m.x), word_unord<kBf16>(m.y), word_unord<kBf16>(m.z),
                        word_unord<kBf16>(m.w));
}

// Same reduction for rows whose byte length is not a multiple of 16: one thread
// per (coarse voxel, element).
template <typename E, bool kBf16>
__global__ void k_ds_amax_elem(const int32_t* __restrict__ seg, const int32_t* __restrict__ srows, int64_t ncoarse,
                               int c, const E* __restrict__ x, E* __restrict__ out) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= ncoarse * c) return;
    const int64_t g = t / c;
    const int ch = (int)(t % c);
    const int32_t s0 = seg[g], s1 = seg[g + 1];
    uint32_t m = 0;
    for (int32_t s = s0; s < s1; ++s) {
        const uint32_t u = (uint32_t)x[(int64_t)srows[s] * c + ch];
        m = max(m, kBf16 ? ord16(u) : ord32(u));
    }
    out[t] = (E)(kBf16 ? unord16(m) : unord32(m));
}

// out[i] = x_coarse[parent[i]] (cache-paired upsampling), one thread per
// (fine voxel, vector of V).
template <typename V>
__global__ void k_gather_rows(const int32_t* __restrict__ parent, int64_t n, int vecs, const V* __restrict__ src,
                              V* __restrict__ dst) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n * vecs) return;
    const int64_t i = t / vecs;
    const int q = (int)(t % vecs);
    dst[t] = src[(int64_t)parent[i] * vecs + q];
}

// Subdivision: output row 8 i + c is child c = 4 ox + 2 oy + oz of voxel i at
// (b, 2x + ox, 2y + oy, 2z + oz), carrying the voxel's features.
__global__ void k_sub_coords(const int4* __restrict__ coords, int64_t n, int4* __restrict__ out) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n * 8) return;
    const int4 c = coords[t >> 3];
    const int o = (int)(t & 7);
    out[t] = make_int4(c.x, 2 * c.y + (o >> 2), 2 * c.z + ((o >> 1) & 1), 2 * c.w + (o & 1));
}

template <typename V>
__global__ void k_sub_feats(int64_t n, int vecs, const V* __restrict__ src, V* __restrict__ dst) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n * 8 * vecs) return;
    const int64_t o = t / vecs;
    const int q = (int)(t % vecs);
    dst[t] = src[(o >> 3) * vecs + q];
}

__global__ void k_check_coords(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez,
                               unsigned int* __restrict__ err) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int4 c = coords[i];
    if ((unsigned)c.x > 65535u || (unsigned)c.y >= (unsigned)ex || (unsigned)c.z >= (unsigned)ey ||
        (unsigned)c.w >= (unsigned)ez)
        atomicOr(err, kErrCoordRange);
}

unsigned grid_for(int64_t work, int threads) { return (unsigned)((work + threads - 1) / threads); }

template <typename V>
cudaError_t launch_rows_copy(bool subdivide, const int32_t* parent, int64_t n, int64_t row_bytes, const void* src,
                             void* dst, cudaStream_t stream) {
    const int vecs = (int)(row_bytes / sizeof(V));
    const int threads = 256;
    if (subdivide) {
        k_sub_feats<V><<<grid_for(n * 8 * vecs, threads), threads, 0, stream>>>(
            n, vecs, static_cast<const V*>(src), static_cast<V*>(dst));
    } else {
        k_gather_rows<V><<<grid_for(n * vecs, threads), threads, 0, stream>>>(
            parent, n, vecs, static_cast<const V*>(src), static_cast<V*>(dst));
    }
    return cudaGetLastError();
}

cudaError_t rows_copy(bool subdivide, const int32_t* parent, int64_t n, int64_t row_bytes, const void* src,
                      void* dst, cudaStream_t stream) {
    if (row_bytes % 16 == 0) return launch_rows_copy<uint4>(subdivide, parent, n, row_bytes, src, dst, stream);
    if (row_bytes % 4 == 0) return launch_rows_copy<uint32_t>(subdivide, parent, n, row_bytes, src, dst, stream);
    return launch_rows_copy<uint16_t>(subdivide, parent, n, row_bytes, src, dst, stream);
}

}  // namespace

int64_t ds_scan_blocks(int64_t n) { return (n + kScanBlock - 1) / kScanBlock; }

int ds_key_bits(const int32_t coarse_extent[3]) {
    return 16 + bits_of(coarse_extent[0]) + bits_of(coarse_extent[1]) + bits_of(coarse_extent[2]);
}

cudaError_t launch_ds_build(const int32_t* coords, int64_t n, const int32_t extent[3], int factor,
                            const int32_t coarse_extent[3], uint64_t* keys[2], int32_t* vals[2], uint32_t* hist,
                            uint32_t* counts, unsigned int* err, int32_t** srows_out, int4* coarse, int32_t* seg,
                            int32_t* parent, cudaStream_t stream) {
    *srows_out = nullptr;
    if (n == 0) return cudaSuccess;
    const CoarseBits kb{bits_of(coarse_extent[2]), bits_of(coarse_extent[1]), bits_of(coarse_extent[0])};
    const int threads = 256;
    k_ds_pack<<<grid_for(n, threads), threads, 0, stream>>>(reinterpret_cast<const int4*>(coords), n, extent[0],
                                                            extent[1], extent[2], factor, kb,
                                                            reinterpret_cast<unsigned long long*>(keys[0]), err);
    int which = 0;
    cudaError_t e = radix_sort_pairs64(keys, nullptr, vals, n, ds_key_bits(coarse_extent), hist, &which, stream);
    if (e != cudaSuccess) return e;
    const auto* sk = reinterpret_cast<const unsigned long long*>(keys[which]);
    const int64_t blocks = ds_scan_blocks(n);
    k_ds_count<<<(unsigned)blocks, 256, 0, stream>>>(sk, n, counts);
    k_ds_scan<<<1, 1024, 0, stream>>>(counts, blocks);
    k_ds_emit<<<(unsigned)blocks, kScanBlock, 0, stream>>>(sk, vals[which], n, kb, counts, coarse, seg, parent);
    *srows_out = vals[which];
    return cudaGetLastError();
}

cudaError_t launch_ds_amax(const int32_t* seg, const int32_t* srows, int64_t ncoarse, bool bf16, int c,
                           const void* x, void* out, cudaStream_t stream) {
    if (ncoarse == 0) return cudaSuccess;
    const int64_t row_bytes = (int64_t)c * (bf16 ? 2 : 4);
    const int threads = 256;
    if (row_bytes % 16 == 0) {
        const int chunks = (int)(row_bytes / 16);
        if (bf16) {
            k_ds_amax<true><<<grid_for(ncoarse * chunks, threads), threads, 0, stream>>>(
                seg, srows, ncoarse, chunks, static_cast<const uint4*>(x), static_cast<uint4*>(out));
        } else {
            k_ds_amax<false><<<grid_for(ncoarse * chunks, threads), threads, 0, stream>>>(
                seg, srows, ncoarse, chunks, static_cast<const uint4*>(x), static_cast<uint4*>(out));
        }
    } else if (bf16) {
        k_ds_amax_elem<uint16_t, true><<<grid_for(ncoarse * c, threads), threads, 0, stream>>>(
            seg, srows, ncoarse, c, static_cast<const uint16_t*>(x), static_cast<uint16_t*>(out));
    } else {
        k_ds_amax_elem<uint32_t, false><<<grid_for(ncoarse * c, threads), threads, 0, stream>>>(
            seg, srows, ncoarse, c, static_cast<const uint32_t*>(x), static_cast<uint32_t*>(out));
    }
    return cudaGetLastError();
}

cudaError_t launch_upsample(const int32_t* parent, int64_t n, int64_t row_bytes, const void* xc, void* out,
                            cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    return rows_copy(false, parent, n, row_bytes, xc, out, stream);
}

cudaError_t launch_subdivide(const int32_t* coords, int64_t n, const int32_t extent[3], int64_t row_bytes,
                             const void* x, int32_t* coords_out, void* x_out, unsigned int* err,
                             cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    k_check_coords<<<grid_for(n, threads), threads, 0, stream>>>(reinterpret_cast<const int4*>(coords), n,
                                                                 extent[0], extent[1], extent[2], err);
    k_sub_coords<<<grid_for(n * 8, threads), threads, 0, stream>>>(reinterpret_cast<const int4*>(coords), n,
                                                                   reinterpret_cast<int4*>(coords_out));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !x || row_bytes == 0) return e;
    return rows_copy(true, nullptr, n, row_bytes, x, x_out, stream);
}

}  // namespace spconv
