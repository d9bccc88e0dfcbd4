// Neighbour-map build on the GPU: pack + validate + hash insert, then probe.
//
// The pages build a map of active voxel coordinates first and probe it per
// kernel offset (trellis-mac article, sparse 3D convolution as gather-scatter,
// step one of its flowchart); the lato.2_mrp_mlx README ("Fleet benchmark")
// caches the resulting index per coordinate set.  Here the map is an
// open-addressing hash table over 64-bit packed keys, built and probed by the
// kernels below, and the probe writes a dense [n, 27] index map with -1 holes.
#include "common.cuh"

namespace spconv {
namespace {

constexpr unsigned long long kEmptyKey = ~0ull;  // never a valid key: coords < 65535

__device__ __forceinline__ unsigned long long pack_key(unsigned b, unsigned x, unsigned y, unsigned z) {
    return ((unsigned long long)b << 48) | ((unsigned long long)x << 32) | ((unsigned long long)y << 16) |
           (unsigned long long)z;
}

// Slot hash: the finaliser of SplitMix64 (Steele, Lea and Flood, "Fast
// splittable pseudorandom number generators", OOPSLA 2014).
__device__ __forceinline__ unsigned long long mix64(unsigned long long k) {
    k ^= k >> 30;
    k *= 0xbf58476d1ce4e5b9ull;
    k ^= k >> 27;
    k *= 0x94d049bb133111ebull;
    k ^= k >> 31;
    return k;
}

// Table layout: slot s occupies two 64-bit words, table[2s] = key and
// table[2s+1] = row index, so one 16-byte load reads a whole slot.
__global__ void k_insert(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez,
                         unsigned long long* __restrict__ table, unsigned long long mask,
                         BuildFlags* __restrict__ flags) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int4 c = coords[i];
    if ((unsigned)c.x > 65535u || (unsigned)c.y >= (unsigned)ex || (unsigned)c.z >= (unsigned)ey ||
        (unsigned)c.w >= (unsigned)ez) {
        atomicOr(&flags->err, kErrCoordRange);
        return;
    }
    const unsigned long long key = pack_key(c.x, c.y, c.z, c.w);
    unsigned long long slot = mix64(key) & mask;
    for (unsigned long long it = 0; it <= mask; ++it) {
        const unsigned long long prev = atomicCAS(&table[2 * slot], kEmptyKey, key);
        if (prev == kEmptyKey) {
            table[2 * slot + 1] = (unsigned long long)i;
            return;
        }
        if (prev == key) {
            atomicOr(&flags->err, kErrDuplicate);
            return;
        }
        slot = (slot + 1) & mask;
    }
    atomicOr(&flags->err, kErrTableFull);
}

// One thread per (voxel i, offset k), k fastest, so the [n, 27] stores coalesce.
__global__ void k_probe(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez,
                        const ulonglong2* __restrict__ table, unsigned long long mask,
                        int32_t* __restrict__ nbr, BuildFlags* __restrict__ flags) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    bool hit = false;
    if (t < n * kVol3) {
        const int64_t i = t / kVol3;
        const int k = (int)(t - i * kVol3);
        int32_t found = -1;
        if (k == kCentre) {
            found = (int32_t)i;
        } else {
            const int4 c = coords[i];
            const int x = c.y + k / 9 - 1, y = c.z + (k / 3) % 3 - 1, z = c.w + k % 3 - 1;
            if ((unsigned)x < (unsigned)ex && (unsigned)y < (unsigned)ey && (unsigned)z < (unsigned)ez) {
                const unsigned long long key = pack_key(c.x, x, y, z);
                unsigned long long slot = mix64(key) & mask;
                for (unsigned long long it = 0; it <= mask; ++it) {
                    const ulonglong2 s = table[slot];
                    if (s.x == key) {
                        found = (int32_t)s.y;
                        break;
                    }
                    if (s.x == kEmptyKey) break;
                    slot = (slot + 1) & mask;
                }
            }
        }
        nbr[t] = found;
        hit = found >= 0;
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, hit);
    if ((threadIdx.x & 31) == 0 && ballot) atomicAdd(&flags->pairs, (unsigned long long)__popc(ballot));
}

}  // namespace

cudaError_t launch_build_map(const int32_t* coords, int64_t n, const int32_t extent[3], int32_t kernel_size,
                             unsigned long long* table, uint64_t slots, int32_t* nbr, BuildFlags* flags,
                             cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(table, 0xFF, slots * 16, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(flags, 0, sizeof(BuildFlags), stream);
    if (e != cudaSuccess) return e;
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const auto* c4 = reinterpret_cast<const int4*>(coords);
    k_insert<<<(unsigned)((n + threads - 1) / threads), threads, 0, stream>>>(
        c4, n, extent[0], extent[1], extent[2], table, slots - 1, flags);
    e = cudaGetLastError();
    if (e != cudaSuccess || kernel_size == 1) return e;
    const int64_t work = n * kVol3;
    k_probe<<<(unsigned)((work + threads - 1) / threads), threads, 0, stream>>>(
        c4, n, extent[0], extent[1], extent[2], reinterpret_cast<const ulonglong2*>(table), slots - 1, nbr,
        flags);
    return cudaGetLastError();
}

}  // namespace spconv

// ---------------------------------------------------------------------------
// Tile metadata.  One CTA per tile stages the tile's [rows, 27] map rows in
// shared memory (coalesced), then warps scan the (offset, class) units with
// ballots: k_tile_count writes the per-unit counts and the tile's padded entry
// total; k_tile_scan turns the totals into offsets; k_tile_fill writes the
// entries (local row, neighbour row) in unit order, rows ascending per unit.
namespace spconv {
namespace {

constexpr int kMetaThreads = 256;

__device__ __forceinline__ void stage_tile_rows(const int32_t* __restrict__ nbr, int64_t row0, int t_eff,
                                                int32_t* __restrict__ tile_s) {
    const int words = t_eff * kVol3;
    const int32_t* src = nbr + row0 * kVol3;
    for (int i = threadIdx.x; i < words; i += blockDim.x) tile_s[i] = __ldg(src + i);
}

__device__ __forceinline__ int unit_offset(int u) {
    const int ks = u / kTileClasses;
    return ks < kCentre ? ks : ks + 1;
}

__global__ void k_tile_count(const int32_t* __restrict__ nbr, int64_t n, int tile_rows,
                             int32_t* __restrict__ tile_counts, int64_t* __restrict__ tile_total) {
    __shared__ int32_t tile_s[kTileRows * kVol3];
    __shared__ int32_t cnt_s[kTileUnits];
    const int64_t t = blockIdx.x;
    const int64_t row0 = t * tile_rows;
    const int t_eff = (int)min((int64_t)tile_rows, n - row0);
    stage_tile_rows(nbr, row0, t_eff, tile_s);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int u = warp; u < kTileUnits; u += kMetaThreads / 32) {
        const int k = unit_offset(u), c = u % kTileClasses;
        int count = 0;
        for (int base = 0; base < kTileRows / kTileClasses; base += 32) {
            const int r = c + kTileClasses * (base + lane);
            const bool hit = r < t_eff && tile_s[r * kVol3 + k] >= 0;
            count += __popc(__ballot_sync(0xffffffffu, hit));
        }
        if (lane == 0) cnt_s[u] = count;
    }
    __syncthreads();
    if (threadIdx.x < kTileCountStride)
        tile_counts[t * kTileCountStride + threadIdx.x] = threadIdx.x < kTileUnits ? cnt_s[threadIdx.x] : 0;
    if (threadIdx.x == 0) {
        int64_t total = 0;
        for (int u = 0; u < kTileUnits; ++u) total += cnt_s[u];
        tile_total[t] = (total + kTileEntryAlign - 1) / kTileEntryAlign * kTileEntryAlign;
    }
}

// Exclusive scan of the per-tile totals (in place, one CTA): off[t] = sum of
// totals before t; off[ntiles] = grand total; off[ntiles + 1] = largest total
// of one tile (the forward kernel sizes its shared-memory entry lists by it).
__global__ void k_tile_scan(int64_t* __restrict__ off, int64_t ntiles) {
    __shared__ int64_t part[1024];
    __shared__ int64_t pmax[1024];
    const int64_t per = (ntiles + blockDim.x - 1) / blockDim.x;
    const int64_t lo = threadIdx.x * per, hi = min(ntiles, lo + per);
    int64_t sum = 0, mx = 0;
    for (int64_t i = lo; i < hi; ++i) {
        sum += off[i];
        mx = max(mx, off[i]);
    }
    part[threadIdx.x] = sum;
    pmax[threadIdx.x] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t run = 0, m = 0;
        for (int i = 0; i < (int)blockDim.x; ++i) {
            const int64_t v = part[i];
            part[i] = run;
            run += v;
            m = max(m, pmax[i]);
        }
        off[ntiles] = run;
        off[ntiles + 1] = m;
    }
    __syncthreads();
    int64_t run = part[threadIdx.x];
    for (int64_t i = lo; i < hi; ++i) {
        const int64_t v = off[i];
        off[i] = run;
        run += v;
    }
}

__global__ void k_tile_fill(const int32_t* __restrict__ nbr, int64_t n, int tile_rows,
                            const int32_t* __restrict__ tile_counts,
                            const int64_t* __restrict__ tile_off, uint16_t* __restrict__ pair_r,
                            int32_t* __restrict__ pair_j) {
    __shared__ int32_t tile_s[kTileRows * kVol3];
    __shared__ int32_t start_s[kTileUnits];
    const int64_t t = blockIdx.x;
    const int64_t row0 = t * tile_rows;
    const int t_eff = (int)min((int64_t)tile_rows, n - row0);
    stage_tile_rows(nbr, row0, t_eff, tile_s);
    if (threadIdx.x == 0) {
        int run = 0;
        for (int u = 0; u < kTileUnits; ++u) {
            start_s[u] = run;
            run += tile_counts[t * kTileCountStride + u];
        }
        // zero the padding entries of this tile
        const int64_t end = tile_off[t + 1];
        for (int64_t e = tile_off[t] + run; e < end; ++e) {
            pair_r[e] = 0;
            pair_j[e] = 0;
        }
    }
    __syncthreads();
    const int64_t base = tile_off[t];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int u = warp; u < kTileUnits; u += kMetaThreads / 32) {
        const int k = unit_offset(u), c = u % kTileClasses;
        int pos = start_s[u];
        for (int b = 0; b < kTileRows / kTileClasses; b += 32) {
            const int r = c + kTileClasses * (b + lane);
            const int32_t j = r < t_eff ? tile_s[r * kVol3 + k] : -1;
            const unsigned m = __ballot_sync(0xffffffffu, j >= 0);
            if (j >= 0) {
                const int64_t e = base + pos + __popc(m & ((1u << lane) - 1u));
                pair_r[e] = (uint16_t)r;
                pair_j[e] = j;
            }
            pos += __popc(m);
        }
    }
}

}  // namespace

cudaError_t launch_tile_count(const int32_t* nbr, int64_t n, int tile_rows, int32_t* tile_counts, int64_t* tile_off,
                              cudaStream_t stream) {
    if (tile_rows < 1 || tile_rows > kTileRows) return cudaErrorInvalidValue;
    const int64_t nt = num_tiles(n, tile_rows);
    if (nt == 0) return cudaMemsetAsync(tile_off, 0, 2 * sizeof(int64_t), stream);
    k_tile_count<<<(unsigned)nt, kMetaThreads, 0, stream>>>(nbr, n, tile_rows, tile_counts, tile_off);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_tile_scan<<<1, 1024, 0, stream>>>(tile_off, nt);
    return cudaGetLastError();
}

cudaError_t launch_tile_fill(const int32_t* nbr, int64_t n, int tile_rows, const int32_t* tile_counts,
                             const int64_t* tile_off, uint16_t* pair_r, int32_t* pair_j, cudaStream_t stream) {
    if (tile_rows < 1 || tile_rows > kTileRows) return cudaErrorInvalidValue;
    const int64_t nt = num_tiles(n, tile_rows);
    if (nt == 0) return cudaSuccess;
    k_tile_fill<<<(unsigned)nt, kMetaThreads, 0, stream>>>(nbr, n, tile_rows, tile_counts, tile_off, pair_r, pair_j);
    return cudaGetLastError();
}

}  // namespace spconv
