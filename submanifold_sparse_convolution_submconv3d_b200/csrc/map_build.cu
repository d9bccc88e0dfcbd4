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
