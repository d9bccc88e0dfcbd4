// Stable least-significant-digit radix sort of (uint32 key, int32 value) pairs on
// the GPU, used by the map build to order the rows by neighbour pattern.
//
// Each pass sorts by one 9-bit digit in three kernels:
//   k_rs_hist     per-block digit counts over a chunk of kRsChunk elements,
//                 written digit-major: hist[digit * nblocks + block];
//   k_rs_scan     one CTA turns the counts into exclusive offsets (digit-major
//                 order, so every block's elements of a digit follow the previous
//                 blocks' elements of that digit);
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

__global__ void k_rs_hist(const uint32_t* __restrict__ keys, int64_t n, int shift, uint32_t* __restrict__ hist) {
    __shared__ uint32_t h[kRsDigits];
    for (int d = threadIdx.x; d < kRsDigits; d += kRsThreads) h[d] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kRsChunk;
    for (int e = threadIdx.x; e < kRsChunk; e += kRsThreads) {
        const int64_t i = base + e;
        if (i < n) atomicAdd(&h[(keys[i] >> shift) & (kRsDigits - 1)], 1u);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < kRsDigits; d += kRsThreads) hist[(int64_t)d * gridDim.x + blockIdx.x] = h[d];
}

// Exclusive scan of `total` counts in place, one CTA of 1024 threads: each thread
// sums a contiguous segment, the segment sums are scanned, then each thread
// rewrites its segment.
__global__ void k_rs_scan(uint32_t* __restrict__ hist, int64_t total) {
    __shared__ uint32_t part[1024];
    const int64_t per = (total + blockDim.x - 1) / blockDim.x;
    const int64_t lo = threadIdx.x * per, hi = min(total, lo + per);
    uint32_t sum = 0;
    for (int64_t i = lo; i < hi; ++i) sum += hist[i];
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int d = 1; d < (int)blockDim.x; d <<= 1) {
        const uint32_t v = threadIdx.x >= (unsigned)d ? part[threadIdx.x - d] : 0u;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    uint32_t run = part[threadIdx.x] - sum;  // exclusive
    for (int64_t i = lo; i < hi; ++i) {
        const uint32_t v = hist[i];
        hist[i] = run;
        run += v;
    }
}

__global__ void __launch_bounds__(kRsThreads) k_rs_scatter(const uint32_t* __restrict__ kin, const int32_t* __restrict__ vin,
                                                           uint32_t* __restrict__ kout, int32_t* __restrict__ vout,
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
        const uint32_t key = valid ? kin[i] : 0u;
        const int32_t val = valid ? (vin ? vin[i] : (int32_t)i) : 0;
        const uint32_t d = (key >> shift) & (kRsDigits - 1);
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

}  // namespace

int64_t radix_hist_words(int64_t n) {
    const int64_t blocks = (n + kRsChunk - 1) / kRsChunk;
    return (blocks > 0 ? blocks : 1) * kRsDigits;
}

cudaError_t radix_sort_pairs(uint32_t* keys[2], const int32_t* vals_in, int32_t* vals[2], int64_t n, int key_bits,
                             uint32_t* hist, int* which, cudaStream_t stream) {
    *which = 0;
    if (n <= 0) return cudaSuccess;
    if (n > 0xFFFFFFFFll) return cudaErrorInvalidValue;
    const unsigned blocks = (unsigned)((n + kRsChunk - 1) / kRsChunk);
    const int passes = key_bits <= 0 ? 1 : (key_bits + kRsBits - 1) / kRsBits;
    int src = 0;
    for (int p = 0; p < passes; ++p) {
        const int shift = p * kRsBits;
        k_rs_hist<<<blocks, kRsThreads, 0, stream>>>(keys[src], n, shift, hist);
        k_rs_scan<<<1, 1024, 0, stream>>>(hist, (int64_t)blocks * kRsDigits);
        // the first pass reads vals_in (the element indices when it is null)
        k_rs_scatter<<<blocks, kRsThreads, 0, stream>>>(keys[src], p == 0 ? vals_in : vals[src], keys[src ^ 1],
                                                        vals[src ^ 1], n, shift, hist);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        src ^= 1;
    }
    *which = src;
    return cudaSuccess;
}

}  // namespace spconv
