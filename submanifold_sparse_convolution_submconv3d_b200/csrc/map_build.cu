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

// Rank of a mask in the reflected Gray-code sequence (the inverse Gray code):
// sorting by it puts masks that differ in few bits next to each other.
__device__ __forceinline__ uint32_t gray_rank(uint32_t g) {
    g ^= g >> 1;
    g ^= g >> 2;
    g ^= g >> 4;
    g ^= g >> 8;
    g ^= g >> 16;
    return g;
}

constexpr int kProbeThreads = 128;

// One thread per voxel: its coordinate is read once and its 26 neighbours are
// probed in turn.  The [rows, 27] results are staged in shared memory so the
// block's stores to the map are contiguous.  Optionally writes the sort key of
// the row: the Gray rank of its 26 non-centre hit bits (offset k, centre
// skipped, is bit 25 - ks with ks = k < 13 ? k : k - 1).
__global__ void __launch_bounds__(kProbeThreads)
    k_probe_rows(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez,
                 const ulonglong2* __restrict__ table, unsigned long long mask, int32_t* __restrict__ nbr,
                 uint32_t* __restrict__ keys, BuildFlags* __restrict__ flags) {
    __shared__ int32_t stage[kProbeThreads * kVol3];
    const int64_t i0 = (int64_t)blockIdx.x * kProbeThreads;
    const int64_t i = i0 + threadIdx.x;
    uint32_t bits = 0;
    int hits = 0;
    if (i < n) {
        const int4 c = coords[i];
        for (int k = 0; k < kVol3; ++k) {
            int32_t found = -1;
            if (k == kCentre) {
                found = (int32_t)i;
            } else {
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
                if (found >= 0) bits |= 1u << (25 - (k < kCentre ? k : k - 1));
            }
            hits += found >= 0 ? 1 : 0;
            stage[threadIdx.x * kVol3 + k] = found;
        }
        if (keys) keys[i] = gray_rank(bits);
    }
    __syncthreads();
    const int rows = (int)min((int64_t)kProbeThreads, n - i0);
    for (int e = threadIdx.x; e < rows * kVol3; e += kProbeThreads) nbr[i0 * kVol3 + e] = stage[e];
    for (int d = 16; d > 0; d >>= 1) hits += __shfl_down_sync(0xffffffffu, hits, d);
    if ((threadIdx.x & 31) == 0 && hits) atomicAdd(&flags->pairs, (unsigned long long)hits);
}

}  // namespace

cudaError_t launch_build_map(const int32_t* coords, int64_t n, const int32_t extent[3], int32_t kernel_size,
                             unsigned long long* table, uint64_t slots, int32_t* nbr, uint32_t* keys,
                             BuildFlags* flags, cudaStream_t stream) {
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
    k_probe_rows<<<(unsigned)((n + kProbeThreads - 1) / kProbeThreads), kProbeThreads, 0, stream>>>(
        c4, n, extent[0], extent[1], extent[2], reinterpret_cast<const ulonglong2*>(table), slots - 1, nbr, keys,
        flags);
    return cudaGetLastError();
}

}  // namespace spconv
