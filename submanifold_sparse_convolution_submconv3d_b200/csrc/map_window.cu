// Window-kernel metadata, built once per coordinate set after the dense map.
//
// The pages fuse the 27 taps into one [N, 27*Cin] x [27*Cin, Cout] matmul over a
// cached device index (lato.2_mrp_mlx README, "Fleet benchmark" and the
// optimisation table after it).  On tcgen05 a matmul's output columns are
// contiguous, so a tap's rows are multiplied in runs of consecutive output rows
// and the holes inside a run cost MMA columns.  The build therefore
//   1. sorts the rows by the Gray rank of their neighbour mask (radix_sort.cu),
//      so rows with similar neighbour patterns are adjacent;
//   2. writes the neighbour table in sorted order and offset-major layout
//      (k_win_permute), so a run's source rows are contiguous in memory;
//   3. covers, per tile and offset, the 16-row windows holding a hit with spans
//      of consecutive windows (k_win_spans), choosing the cover that costs the
//      tensor pipe least: a tcgen05.mma with M = 128 and K = 16 costs the same
//      few dozen cycles for any N up to about 112 columns and N / 2 cycles above
//      that (measured on B200), so a span costs max(floor, windows) and merging
//      nearby windows into one span is free up to the floor;
//   4. concatenates, per tile, the source rows of all its jobs in job order
//      (k_win_stream), so the forward fetches a tile's indices in one copy;
//   5. orders the tiles by estimated cost, most expensive first (k_win_cost and
//      the radix sort), the order in which the forward's CTAs claim them.
#include "common.cuh"

namespace spconv {
namespace {

constexpr int kFloorWindows = 7;  // windows of 16 columns that one MMA issue costs at least
constexpr uint32_t kCostKeyMax = 511;  // claim-order keys take 9 bits

// One thread per sorted row r (r < npad): perm[r] = the row it holds and
// nbr_t[k * npad + r] = that row's neighbour at offset k (-1 for padding rows).
__global__ void k_win_permute(const int32_t* __restrict__ nbr, const int32_t* __restrict__ sorted_rows, int64_t n,
                              int64_t npad, int32_t* __restrict__ perm, int32_t* __restrict__ nbr_t) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= npad) return;
    if (r < n) {
        const int32_t i = sorted_rows[r];
        perm[r] = i;
        const int32_t* row = nbr + (int64_t)i * kVol3;
#pragma unroll
        for (int k = 0; k < kVol3; ++k) nbr_t[k * npad + r] = row[k];
    } else {
#pragma unroll
        for (int k = 0; k < kVol3; ++k) nbr_t[k * npad + r] = -1;
    }
}

// Cheapest cover of the set windows of `occ` (w windows) by spans of consecutive
// windows, each span costing max(kFloorWindows, its windows); ties go to fewer
// covered windows.  Writes spans as (first window, windows) in increasing order.
__device__ int cover_spans(uint32_t occ, int w, uint32_t* spans) {
    int best[kWinMaxRows / kWinCols + 1];
    int from[kWinMaxRows / kWinCols + 1];
    best[0] = 0;
    for (int i = 1; i <= w; ++i) {
        if (!((occ >> (i - 1)) & 1u)) {  // an empty window ends no span
            best[i] = best[i - 1];
            from[i] = -1;
            continue;
        }
        best[i] = 0x7fffffff;
        from[i] = i - 1;
        for (int j = i - 1; j >= 0; --j) {  // span covers windows j .. i-1
            const int len = i - j;
            const int c = best[j] + (len > kFloorWindows ? len : kFloorWindows) * 64 + len;
            if (c < best[i]) {
                best[i] = c;
                from[i] = j;
            }
        }
    }
    uint32_t rev[kWinMaxSpans];
    int ns = 0;
    for (int i = w; i > 0;) {
        if (from[i] < 0) {
            --i;
            continue;
        }
        if (ns < kWinMaxSpans) rev[ns] = ((uint32_t)from[i] << 8) | (uint32_t)(i - from[i]);
        ++ns;
        i = from[i];
    }
    for (int s = 0; s < ns && s < kWinMaxSpans; ++s) spans[s] = rev[ns - 1 - s];
    return ns;
}

// One warp per tile: window occupancy of the 26 non-centre offsets by ballots,
// then lane j covers offset j's windows, and the spans are compacted into the
// tile's job list after the centre job.  The offset order is rotated per tile so
// that tiles processed at the same time ask L2 for different weight tiles.
__global__ void k_win_spans(const int32_t* __restrict__ nbr_t, int64_t npad, int rows, int64_t tiles,
                            uint32_t* __restrict__ jobs, int64_t* __restrict__ tile_cols,
                            BuildFlags* __restrict__ flags) {
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= tiles) return;  // whole warps exit together
    const int w = rows / kWinCols;
    const int rot = (int)(t % (kVol3 - 1));
    uint32_t my_occ = 0;
    for (int j = 0; j < kVol3 - 1; ++j) {
        const int ks = (j + rot) % (kVol3 - 1);
        const int k = ks < kCentre ? ks : ks + 1;
        const int32_t* col = nbr_t + (int64_t)k * npad + t * rows;
        uint32_t occ = 0;
        for (int base = 0; base < rows; base += 32) {
            const bool hit = base + lane < rows && col[base + lane] >= 0;
            const uint32_t b = __ballot_sync(0xffffffffu, hit);
            if (b & 0xFFFFu) occ |= 1u << (base / kWinCols);
            if (b >> 16) occ |= 1u << (base / kWinCols + 1);
        }
        if (lane == j) my_occ = occ;
    }
    uint32_t spans[kWinMaxSpans];
    int ns = 0;
    int cols = 0;
    if (lane < kVol3 - 1 && my_occ) {
        ns = cover_spans(my_occ, w, spans);
        if (ns > kWinMaxSpans) {  // cannot happen: spans are separated by empty windows
            atomicOr(&flags->err, kErrInternal);
            ns = kWinMaxSpans;
        }
        for (int s = 0; s < ns; ++s) cols += (int)(spans[s] & 255u) * kWinCols;
    }
    int incl = ns;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t* tj = jobs + t * kWinJobStride;
    const int ks = (lane + rot) % (kVol3 - 1);
    const int k = ks < kCentre ? ks : ks + 1;
    for (int s = 0; s < ns; ++s)
        tj[kWinRecHeader + 1 + incl - ns + s] = win_job(k, (int)(spans[s] >> 8), (int)(spans[s] & 255u));
    if (lane == 0) {
        tj[0] = (uint32_t)(1 + total);
        tj[kWinRecHeader] = win_job(kCentre, 0, w);
    }
    for (int d = 16; d > 0; d >>= 1) cols += __shfl_down_sync(0xffffffffu, cols, d);
    if (lane == 0) {
        atomicAdd(&flags->spans, (unsigned long long)total);
        atomicAdd(&flags->span_cols, (unsigned long long)cols);
        tile_cols[t] = rows + cols;  // the tile's index-stream length: centre job + spans
        atomicMax(&flags->max_tile_cols, (unsigned long long)(rows + cols));
    }
}

// Exclusive scan of the per-tile stream lengths, in place, one CTA of 1024
// threads; off[tiles] receives the total.
__global__ void k_win_scan(int64_t* __restrict__ off, int64_t tiles) {
    __shared__ int64_t part[1024];
    const int64_t per = (tiles + blockDim.x - 1) / blockDim.x;
    const int64_t lo = threadIdx.x * per, hi = min(tiles, lo + per);
    int64_t sum = 0;
    for (int64_t i = lo; i < hi; ++i) sum += off[i];
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int d = 1; d < (int)blockDim.x; d <<= 1) {
        const int64_t v = threadIdx.x >= (unsigned)d ? part[threadIdx.x - d] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int64_t run = part[threadIdx.x] - sum;
    for (int64_t i = lo; i < hi; ++i) {
        const int64_t v = off[i];
        off[i] = run;
        run += v;
    }
    if (threadIdx.x == blockDim.x - 1) off[tiles] = part[threadIdx.x];
}

// One warp per tile: the tile's index stream is every job's source rows, job
// after job (centre first), so the forward fetches a tile's indices with one
// contiguous copy.
__global__ void k_win_stream(const int32_t* __restrict__ nbr_t, int64_t npad, int rows, int64_t tiles,
                             uint32_t* __restrict__ jobs, const int64_t* __restrict__ off,
                             int32_t* __restrict__ stream) {
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= tiles) return;
    uint32_t* tj = jobs + t * kWinJobStride;
    const int nj = (int)tj[0];
    int64_t pos = off[t];
    if (lane == 0) {  // the record's header: where the tile's stream is
        tj[1] = (uint32_t)(off[t + 1] - pos);
        tj[2] = (uint32_t)((uint64_t)pos & 0xFFFFFFFFu);
        tj[3] = (uint32_t)((uint64_t)pos >> 32);
    }
    for (int j = 0; j < nj; ++j) {
        const uint32_t jw = tj[kWinRecHeader + j];
        const int ncols = win_job_nw(jw) * kWinCols;
        const int32_t* src = nbr_t + (int64_t)win_job_k(jw) * npad + t * rows + win_job_w0(jw) * kWinCols;
        for (int e = lane; e < ncols; e += 32) stream[pos + e] = src[e];
        pos += ncols;
    }
}

// One thread per tile: the sort key of the tile claim order, so the forward's
// CTAs take the most expensive tiles first and finish together.  The cost
// estimate weighs a job's fixed issue overhead against its columns.
__global__ void k_win_cost(const uint32_t* __restrict__ jobs, int64_t tiles, uint32_t* __restrict__ keys) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= tiles) return;
    const uint32_t* tj = jobs + t * kWinJobStride;
    // cost 4 J + stream / 16 is below 2^11 (J <= 209, stream <= 27 * 256); a step of
    // 4 (about one job) keeps the key to one 9-bit radix pass
    const uint32_t cost = (4u * tj[0] + tj[1] / 16u) >> 2;
    keys[t] = kCostKeyMax - (cost < kCostKeyMax ? cost : kCostKeyMax);  // ascending sort = descending cost
}

}  // namespace

cudaError_t launch_win_cost(const uint32_t* jobs, int64_t tiles, uint32_t* keys, cudaStream_t stream) {
    if (tiles <= 0) return cudaSuccess;
    k_win_cost<<<(unsigned)((tiles + 255) / 256), 256, 0, stream>>>(jobs, tiles, keys);
    return cudaGetLastError();
}

cudaError_t launch_win_meta(const int32_t* nbr, const int32_t* sorted_rows, int64_t n, int rows, int64_t tiles,
                            int64_t npad, int32_t* perm, int32_t* nbr_t, uint32_t* jobs, int64_t* idx_off,
                            int32_t* idx_stream, BuildFlags* flags, cudaStream_t stream) {
    if (rows < kWinCols || rows > kWinMaxRows || rows % kWinCols != 0) return cudaErrorInvalidValue;
    if (tiles <= 0) return cudaSuccess;
    const int threads = 256;
    k_win_permute<<<(unsigned)((npad + threads - 1) / threads), threads, 0, stream>>>(nbr, sorted_rows, n, npad, perm,
                                                                                       nbr_t);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t warps_per_block = threads / 32;
    const unsigned warp_blocks = (unsigned)((tiles + warps_per_block - 1) / warps_per_block);
    k_win_spans<<<warp_blocks, threads, 0, stream>>>(nbr_t, npad, rows, tiles, jobs, idx_off, flags);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_win_scan<<<1, 1024, 0, stream>>>(idx_off, tiles);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_win_stream<<<warp_blocks, threads, 0, stream>>>(nbr_t, npad, rows, tiles, jobs, idx_off, idx_stream);
    return cudaGetLastError();
}

}  // namespace spconv
