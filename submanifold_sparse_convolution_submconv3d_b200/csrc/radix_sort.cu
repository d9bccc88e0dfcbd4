// Stable least-significant-digit radix sort of (uint32 or uint64 key, int32 value)
// pairs on the GPU.  The map build uses it to order the rows by neighbour pattern
// and the tiles by cost (32-bit keys), the sorted-key map build and the
// downsample to order packed coordinates (64-bit keys).
//
// Each pass sorts by one 9-bit digit:
//   k_rs_hist     per-block digit counts over a chunk of kRsChunk elements,
//                 written digit-major: hist[digit * nblocks + block];
//   k_scan_*      the counts become exclusive offsets (digit-major order, so
//                 every block's elements of a digit follow the previous blocks'
//                 elements of that digit), by a three-kernel chunked scan;
//   k_rs_scatter  each block walks its chunk in rounds of one element per thread;
//                 within a warp, equal digits are ranked with __match_any_sync,
//                 across warps by a per-digit prefix in shared memory, so elements
//                 keep their input order inside a digit (stable) and the result
//                 is deterministic.
#include "common.cuh"

namespace spconv {
namespace {

constexpr int kRsBits = 9;
constexpr int kRsDigits = 1 << kRsBits;
constexpr int kRsThreads = 256;
constexpr int kRsWarps = kRsThreads / 32;
constexpr int kRsItems = 8;
constexpr int kRsChunk = kRsThreads * kRsItems;  // elements per block

template <typename K>
__global__ void k_rs_hist(const K* __restrict__ keys, int64_t n, int shift, uint32_t* __restrict__ hist) {
    __shared__ uint32_t h[kRsDigits];
    for (int d = threadIdx.x; d < kRsDigits; d += kRsThreads) h[d] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kRsChunk;
    for (int e = threadIdx.x; e < kRsChunk; e += kRsThreads) {
        const int64_t i = base + e;
        if (i < n) atomicAdd(&h[(uint32_t)(keys[i] >> shift) & (kRsDigits - 1)], 1u);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < kRsDigits; d += kRsThreads) hist[(int64_t)d * gridDim.x + blockIdx.x] = h[d];
}

// Exclusive scan of the `total` digit-major counts in place, in three kernels:
// every CTA sums a chunk of kScanChunk counts, one CTA scans the chunk sums, and
// every CTA rescans its chunk from its chunk's offset.
constexpr int kScanThreads = 256;
constexpr int kScanItems = 16;
constexpr int kScanChunk = kScanThreads * kScanItems;

__global__ void __launch_bounds__(kScanThreads) k_scan_reduce(const uint32_t* __restrict__ in, int64_t total,
                                                               uint32_t* __restrict__ partial) {
    const int64_t base = (int64_t)blockIdx.x * kScanChunk;
    uint32_t sum = 0;
    for (int e = threadIdx.x; e < kScanChunk; e += kScanThreads) {
        const int64_t i = base + e;
        if (i < total) sum += in[i];
    }
    for (int d = 16; d > 0; d >>= 1) sum += __shfl_down_sync(0xffffffffu, sum, d);
    __shared__ uint32_t part[kScanThreads / 32];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (int w = 0; w < kScanThreads / 32; ++w) t += part[w];
        partial[blockIdx.x] = t;
    }
}

// One CTA of 1024 threads: exclusive scan of the chunk sums in place.
__global__ void __launch_bounds__(1024) k_scan_partials(uint32_t* __restrict__ partial, int64_t chunks) {
    __shared__ uint32_t part[1024];
    const int64_t per = (chunks + blockDim.x - 1) / blockDim.x;
    const int64_t lo = threadIdx.x * per, hi = min(chunks, lo + per);
    uint32_t sum = 0;
    for (int64_t i = lo; i < hi; ++i) sum += partial[i];
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
        const uint32_t v = partial[i];
        partial[i] = run;
        run += v;
    }
}

// Thread t of a CTA owns kScanItems consecutive counts of the chunk.
__global__ void __launch_bounds__(kScanThreads) k_scan_apply(uint32_t* __restrict__ data, int64_t total,
                                                              const uint32_t* __restrict__ partial) {
    __shared__ uint32_t wsum[kScanThreads / 32];
    const int64_t base = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanItems;
    uint32_t v[kScanItems];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < kScanItems; ++j) {
        v[j] = base + j < total ? data[base + j] : 0u;
        sum += v[j];
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = sum;
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t before = partial[blockIdx.x];
    for (int w = 0; w < warp; ++w) before += wsum[w];
    uint32_t run = before + incl - sum;
#pragma unroll
    for (int j = 0; j < kScanItems; ++j) {
        if (base + j < total) data[base + j] = run;
        run += v[j];
    }
}

template <typename K>
__global__ void __launch_bounds__(kRsThreads) k_rs_scatter(const K* __restrict__ kin, const int32_t* __restrict__ vin,
                                                           K* __restrict__ kout, int32_t* __restrict__ vout,
                                                           int64_t n, int shift, const uint32_t* __restrict__ offs) {
    __shared__ uint32_t next[kRsDigits];            // next output position of each digit for this block
    __shared__ uint32_t wpos[kRsWarps][kRsDigits];  // per round: warp counts, then warp start positions
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int d = threadIdx.x; d < kRsDigits; d += kRsThreads) {
        next[d] = offs[(int64_t)d * gridDim.x + blockIdx.x];
        for (int w = 0; w < kRsWarps; ++w) wpos[w][d] = 0;
    }
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int round = 0; round < kRsItems; ++round) {
        __syncthreads();  // wpos is zeroed (set-up or the end of the previous round)
        const int64_t i = (int64_t)blockIdx.x * kRsChunk + (int64_t)round * kRsThreads + threadIdx.x;
        const bool valid = i < n;
        const K key = valid ? kin[i] : K(0);
        const int32_t val = valid ? (vin ? vin[i] : (int32_t)i) : 0;
        const uint32_t d = (uint32_t)(key >> shift) & (kRsDigits - 1);
        // invalid lanes get a tag no digit can equal, so they never join a group
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? d : (0x80000000u | (uint32_t)lane));
        const int rank = __popc(peers & lt_mask);
        if (valid && rank == 0) wpos[warp][d] = (uint32_t)__popc(peers);
        __syncthreads();
        for (int dd = threadIdx.x; dd < kRsDigits; dd += kRsThreads) {
            uint32_t run = next[dd];
            for (int w = 0; w < kRsWarps; ++w) {
                const uint32_t c = wpos[w][dd];
                wpos[w][dd] = run;
                run += c;
            }
            next[dd] = run;
        }
        __syncthreads();
        if (valid) {
            const uint32_t pos = wpos[warp][d] + (uint32_t)rank;
            kout[pos] = key;
            vout[pos] = val;
        }
        __syncthreads();
        for (int dd = threadIdx.x; dd < kRsDigits; dd += kRsThreads)
            for (int w = 0; w < kRsWarps; ++w) wpos[w][dd] = 0;
    }
}

template <typename K>
cudaError_t sort_pairs(K* keys[2], const int32_t* vals_in, int32_t* vals[2], int64_t n, int key_bits, uint32_t* hist,
                       int* which, cudaStream_t stream) {
    *which = 0;
    if (n <= 0) return cudaSuccess;
    if (n > 0xFFFFFFFFll) return cudaErrorInvalidValue;
    const unsigned blocks = (unsigned)((n + kRsChunk - 1) / kRsChunk);
    const int passes = key_bits <= 0 ? 1 : (key_bits + kRsBits - 1) / kRsBits;
    const int64_t total = (int64_t)blocks * kRsDigits;
    const unsigned chunks = (unsigned)((total + kScanChunk - 1) / kScanChunk);
    uint32_t* partial = hist + total;  // radix_hist_words leaves room for the chunk sums
    int src = 0;
    for (int p = 0; p < passes; ++p) {
        const int shift = p * kRsBits;
        k_rs_hist<K><<<blocks, kRsThreads, 0, stream>>>(keys[src], n, shift, hist);
        k_scan_reduce<<<chunks, kScanThreads, 0, stream>>>(hist, total, partial);
        k_scan_partials<<<1, 1024, 0, stream>>>(partial, chunks);
        k_scan_apply<<<chunks, kScanThreads, 0, stream>>>(hist, total, partial);
        // the first pass reads vals_in (the element indices when it is null)
        k_rs_scatter<K><<<blocks, kRsThreads, 0, stream>>>(keys[src], p == 0 ? vals_in : vals[src], keys[src ^ 1],
                                                           vals[src ^ 1], n, shift, hist);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        src ^= 1;
    }
    *which = src;
    return cudaSuccess;
}

}  // namespace

int64_t radix_hist_words(int64_t n) {
    const int64_t blocks = (n + kRsChunk - 1) / kRsChunk;
    const int64_t total = (blocks > 0 ? blocks : 1) * kRsDigits;
    return total + (total + kScanChunk - 1) / kScanChunk;
}

cudaError_t radix_sort_pairs(uint32_t* keys[2], const int32_t* vals_in, int32_t* vals[2], int64_t n, int key_bits,
                             uint32_t* hist, int* which, cudaStream_t stream) {
    return sort_pairs<uint32_t>(keys, vals_in, vals, n, key_bits, hist, which, stream);
}

cudaError_t radix_sort_pairs64(uint64_t* keys[2], const int32_t* vals_in, int32_t* vals[2], int64_t n, int key_bits,
                               uint32_t* hist, int* which, cudaStream_t stream) {
    return sort_pairs<uint64_t>(keys, vals_in, vals, n, key_bits, hist, which, stream);
}

}  // namespace spconv
