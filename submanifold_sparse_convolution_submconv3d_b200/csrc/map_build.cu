// Neighbour-map build on the GPU: pack + validate, a coordinate dictionary, then
// one probe per voxel and kernel offset.
//
// The pages build a map of active voxel coordinates first and probe it per
// kernel offset (trellis-mac article, sparse 3D convolution as gather-scatter,
// step one of its flowchart); the lato.2_mrp_mlx README ("Fleet benchmark")
// caches the resulting index per coordinate set.  Two dictionaries are built
// here, both writing the same dense [n, 27] index map with -1 holes:
//   - an open-addressing hash table over 64-bit packed keys (the default);
//   - the sorted-key index map that the lato.2_mrp_mlx README's table of
//     upstream equivalents gives for its own port: the packed keys radix-sorted
//     with their rows, each neighbour found by binary search.
// Orientation: the map gathers p + d_k (cross-correlation, as the README's
// "Correctness" section says the port implements) or, with the flip option,
// p - d_k (the alternative the same section leaves open and its --flip-kernel
// switch builds), which is the same map with k and 26 - k exchanged.
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
constexpr int kProbeBatch = 3;  // offsets whose first hash slots one thread loads together

// One thread per voxel: its coordinate is read once and its 26 neighbours are
// probed in turn.  The [rows, 27] results are staged in shared memory so the
// block's stores to the map are contiguous.  Optionally writes the sort key of
// the row: the Gray rank of its 26 non-centre hit bits (offset k, centre
// skipped, is bit 25 - ks with ks = k < 13 ? k : k - 1).
__global__ void __launch_bounds__(kProbeThreads)
    k_probe_rows(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez, int sign,
                 const ulonglong2* __restrict__ table, unsigned long long mask, int32_t* __restrict__ nbr,
                 uint32_t* __restrict__ keys, BuildFlags* __restrict__ flags) {
    __shared__ int32_t stage[kProbeThreads * kVol3];
    const int64_t i0 = (int64_t)blockIdx.x * kProbeThreads;
    const int64_t i = i0 + threadIdx.x;
    uint32_t bits = 0;
    int hits = 0;
    if (i < n) {
        const int4 c = coords[i];
        // the offsets in batches of kProbeBatch: a batch's first slots are loaded
        // together (independent loads), then any probe whose first slot holds
        // another key walks on alone (rare at load factor <= 1/2)
#pragma unroll
        for (int k0 = 0; k0 < kVol3; k0 += kProbeBatch) {
            unsigned long long key[kProbeBatch];
            unsigned long long slot[kProbeBatch];
            bool inside[kProbeBatch];
            ulonglong2 first[kProbeBatch];
#pragma unroll
            for (int q = 0; q < kProbeBatch; ++q) {
                const int k = k0 + q;
                const int x = c.y + sign * (k / 9 - 1), y = c.z + sign * ((k / 3) % 3 - 1),
                          z = c.w + sign * (k % 3 - 1);
                inside[q] = k != kCentre && (unsigned)x < (unsigned)ex && (unsigned)y < (unsigned)ey &&
                            (unsigned)z < (unsigned)ez;
                key[q] = inside[q] ? pack_key(c.x, x, y, z) : kEmptyKey;
                slot[q] = mix64(key[q]) & mask;
                first[q] = inside[q] ? table[slot[q]] : make_ulonglong2(kEmptyKey, 0);
            }
#pragma unroll
            for (int q = 0; q < kProbeBatch; ++q) {
                const int k = k0 + q;
                int32_t found = -1;
                if (k == kCentre) {
                    found = (int32_t)i;
                } else if (inside[q]) {
                    ulonglong2 sv = first[q];
                    unsigned long long sl = slot[q];
                    for (unsigned long long it = 0; it <= mask; ++it) {
                        if (sv.x == key[q]) {
                            found = (int32_t)sv.y;
                            break;
                        }
                        if (sv.x == kEmptyKey) break;
                        sl = (sl + 1) & mask;
                        sv = table[sl];
                    }
                }
                if (k != kCentre && found >= 0) bits |= 1u << (25 - (k < kCentre ? k : k - 1));
                hits += found >= 0 ? 1 : 0;
                stage[threadIdx.x * kVol3 + k] = found;
            }
        }
        if (keys) keys[i] = gray_rank(bits);
    }
    __syncthreads();
    const int rows = (int)min((int64_t)kProbeThreads, n - i0);
    for (int e = threadIdx.x; e < rows * kVol3; e += kProbeThreads) nbr[i0 * kVol3 + e] = stage[e];
    for (int d = 16; d > 0; d >>= 1) hits += __shfl_down_sync(0xffffffffu, hits, d);
    if ((threadIdx.x & 31) == 0 && hits) atomicAdd(&flags->pairs, (unsigned long long)hits);
}

// ---------------------------------------------------------------- sorted keys
// Key of the sorted dictionary: (b, x, y, z) packed into bit fields just wide
// enough for the extents, b in the top 16 bits, so that key order is the
// lexicographic order of (b, x, y, z) and a neighbour's key is the voxel's key
// plus a per-offset constant whenever the neighbour lies inside the grid.
struct KeyBits {
    int bz, by, bx;
};

__device__ __forceinline__ unsigned long long sk_pack(KeyBits kb, unsigned b, unsigned x, unsigned y, unsigned z) {
    return ((unsigned long long)b << (kb.bx + kb.by + kb.bz)) | ((unsigned long long)x << (kb.by + kb.bz)) |
           ((unsigned long long)y << kb.bz) | (unsigned long long)z;
}

// Key step of offset k: sign * (dx << (by + bz) + dy << bz + dz).
__device__ __forceinline__ long long sk_delta(KeyBits kb, int k, int sign) {
    const long long dx = k / 9 - 1, dy = (k / 3) % 3 - 1, dz = k % 3 - 1;
    return sign * (dx * (1ll << (kb.by + kb.bz)) + dy * (1ll << kb.bz) + dz);
}

__global__ void k_sk_pack(const int4* __restrict__ coords, int64_t n, int ex, int ey, int ez, KeyBits kb,
                          unsigned long long* __restrict__ keys, BuildFlags* __restrict__ flags) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int4 c = coords[i];
    if ((unsigned)c.x > 65535u || (unsigned)c.y >= (unsigned)ex || (unsigned)c.z >= (unsigned)ey ||
        (unsigned)c.w >= (unsigned)ez) {
        atomicOr(&flags->err, kErrCoordRange);
        keys[i] = 0;  // the build fails; the key only has to keep the later kernels in bounds
        return;
    }
    keys[i] = sk_pack(kb, c.x, c.y, c.z, c.w);
}

__global__ void k_sk_dups(const unsigned long long* __restrict__ skeys, int64_t n, BuildFlags* __restrict__ flags) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 1 && i < n && skeys[i] == skeys[i - 1]) atomicOr(&flags->err, kErrDuplicate);
}

// First position in [lo, hi) whose key is >= t (upper: > t).
__device__ __forceinline__ int64_t sk_bound(const unsigned long long* __restrict__ skeys, int64_t lo, int64_t hi,
                                            long long t, bool upper) {
    while (lo < hi) {
        const int64_t mid = lo + ((hi - lo) >> 1);
        const long long v = (long long)skeys[mid];
        if (upper ? v <= t : v < t) {
            lo = mid + 1;
        } else {
            hi = mid;
        }
    }
    return lo;
}

// One thread per sorted position.  A block's voxels are consecutive in key
// order, so for each offset their neighbours' keys lie between the first voxel's
// key and the last voxel's key, both shifted by the offset's key step: the block
// first narrows every offset's search to that range of the sorted array (two
// binary searches per offset), then each thread searches its neighbours inside
// the ranges.  Writes the map row of the voxel's own row index and its sort key.
__global__ void __launch_bounds__(kProbeThreads)
    k_sk_probe(const unsigned long long* __restrict__ skeys, const int32_t* __restrict__ srows, int64_t n, int ex,
               int ey, int ez, KeyBits kb, int sign, int32_t* __restrict__ nbr, uint32_t* __restrict__ keys,
               BuildFlags* __restrict__ flags) {
    __shared__ int64_t range[2 * kVol3];
    const int64_t s0 = (int64_t)blockIdx.x * kProbeThreads;
    const int64_t s1 = min(n, s0 + kProbeThreads) - 1;
    if (threadIdx.x < 2 * kVol3) {
        const int k = threadIdx.x >> 1;
        const bool upper = threadIdx.x & 1;
        const long long t = (long long)skeys[upper ? s1 : s0] + sk_delta(kb, k, sign);
        range[threadIdx.x] = sk_bound(skeys, 0, n, t, upper);
    }
    __syncthreads();
    const int64_t s = s0 + threadIdx.x;
    int hits = 0;
    if (s < n) {
        const int32_t r = srows[s];
        const unsigned long long key = skeys[s];
        const int z = (int)(key & ((1ull << kb.bz) - 1));
        const int y = (int)((key >> kb.bz) & ((1ull << kb.by) - 1));
        const int x = (int)((key >> (kb.by + kb.bz)) & ((1ull << kb.bx) - 1));
        uint32_t bits = 0;
        int32_t row[kVol3];
#pragma unroll
        for (int k = 0; k < kVol3; ++k) {
            int32_t found = -1;
            if (k == kCentre) {
                found = r;
            } else {
                const int nx = x + sign * (k / 9 - 1), ny = y + sign * ((k / 3) % 3 - 1), nz = z + sign * (k % 3 - 1);
                if ((unsigned)nx < (unsigned)ex && (unsigned)ny < (unsigned)ey && (unsigned)nz < (unsigned)ez) {
                    const long long t = (long long)key + sk_delta(kb, k, sign);
                    const int64_t hi = range[2 * k + 1];
                    const int64_t pos = sk_bound(skeys, range[2 * k], hi, t, false);
                    if (pos < hi && (long long)skeys[pos] == t) found = srows[pos];
                }
                if (found >= 0) bits |= 1u << (25 - (k < kCentre ? k : k - 1));
            }
            hits += found >= 0 ? 1 : 0;
            row[k] = found;
        }
#pragma unroll
        for (int k = 0; k < kVol3; ++k) nbr[(int64_t)r * kVol3 + k] = row[k];
        if (keys) keys[r] = gray_rank(bits);
    }
    for (int d = 16; d > 0; d >>= 1) hits += __shfl_down_sync(0xffffffffu, hits, d);
    if ((threadIdx.x & 31) == 0 && hits) atomicAdd(&flags->pairs, (unsigned long long)hits);
}

int bits_for(int extent) {
    int b = 0;
    while ((1 << b) < extent) ++b;
    return b;
}

}  // namespace

int sorted_key_bits(const int32_t extent[3]) {
    return 16 + bits_for(extent[0]) + bits_for(extent[1]) + bits_for(extent[2]);
}

cudaError_t launch_build_map(const int32_t* coords, int64_t n, const int32_t extent[3], int32_t kernel_size,
                             unsigned long long* table, uint64_t slots, int32_t* nbr, uint32_t* keys,
                             BuildFlags* flags, cudaStream_t stream, const MapBuildOpts& opts) {
    const int sign = opts.flip ? -1 : 1;
    if (opts.sorted) {
        cudaError_t e = cudaMemsetAsync(flags, 0, sizeof(BuildFlags), stream);
        if (e != cudaSuccess || n == 0) return e;
        const KeyBits kb{bits_for(extent[2]), bits_for(extent[1]), bits_for(extent[0])};
        const int threads = 256;
        const unsigned blocks = (unsigned)((n + threads - 1) / threads);
        const auto* c4 = reinterpret_cast<const int4*>(coords);
        k_sk_pack<<<blocks, threads, 0, stream>>>(c4, n, extent[0], extent[1], extent[2], kb,
                                                  reinterpret_cast<unsigned long long*>(opts.skeys[0]), flags);
        int which = 0;
        uint64_t* skeys[2] = {opts.skeys[0], opts.skeys[1]};
        int32_t* svals[2] = {opts.svals[0], opts.svals[1]};
        e = radix_sort_pairs64(skeys, nullptr, svals, n, sorted_key_bits(extent), opts.hist, &which, stream);
        if (e != cudaSuccess) return e;
        const auto* sk = reinterpret_cast<const unsigned long long*>(opts.skeys[which]);
        k_sk_dups<<<blocks, threads, 0, stream>>>(sk, n, flags);
        if (kernel_size == 1) return cudaGetLastError();
        k_sk_probe<<<(unsigned)((n + kProbeThreads - 1) / kProbeThreads), kProbeThreads, 0, stream>>>(
            sk, opts.svals[which], n, extent[0], extent[1], extent[2], kb, sign, nbr, keys, flags);
        return cudaGetLastError();
    }
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
        c4, n, extent[0], extent[1], extent[2], sign, reinterpret_cast<const ulonglong2*>(table), slots - 1, nbr,
        keys, flags);
    return cudaGetLastError();
}

}  // namespace spconv
