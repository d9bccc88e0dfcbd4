// Fused gather -> tcgen05 GEMM -> single-write store, bf16 in, fp32 accumulate.
//
// The pages fuse the 27 per-offset taps into one [N, 27*Cin] x [27*Cin, Cout]
// matmul over a cached device index (lato.2_mrp_mlx README, "Fleet benchmark"
// and the optimisation table after it).  This kernel computes the same sum, laid
// out for sm_100a:
//
//   D^T[Cout_blk, rows] = sum_k W_k^T[Cout_blk, Cin] . X_k^T[Cin, rows]
//
// One CTA owns kTileRows consecutive output rows and one block of 64 or 128
// output channels.  Tensor memory (TMEM, 128 lanes x 512 fp32 columns) holds
//   * the accumulator: lane = output channel, column = output row of the tile;
//   * two scratch buffers of kScratchCols columns and a few dummy columns.
// The centre offset (every row is its own neighbour) is one dense MMA per 128
// rows straight into the accumulator.  For every other offset the rows of the
// tile that have a neighbour there are compacted into a list; their neighbour
// feature rows are gathered (cp.async, 16 B, zero-filled padding) into a
// swizzled shared-memory tile and multiplied into a scratch buffer, and four
// warps then add each scratch column into the accumulator column of its row
// (tcgen05.ld / tcgen05.st, no atomics).  Weights W_k arrive by TMA.  At the
// end each output row is written exactly once, with bias, rounded to bf16.
//
// Warp roles (576 threads):
//   warp 0      TMA producer of weight tiles (A operand)
//   warp 1      TMEM allocator and tcgen05.mma issuer
//   warps 2-5   gather producers of feature rows (B operand)
//   warps 6-17  scratch -> accumulator fold, then the epilogue: three warps per
//               TMEM lane quarter, each owning the tile rows of one residue mod 3,
//               so no accumulator column is touched by two warps of a quarter.
//               Narrow TMEM accesses are issued without per-element branches;
//               padding entries go to dedicated dummy columns.
// Every spin-wait is bounded: after kWaitTimeoutNs the kernel records
// kFwdErrTimeout in the map's error word, stops issuing work, lets copies in
// flight land, frees its TMEM and returns.
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace spconv {
namespace {

using namespace sm100;

constexpr int kTileRows = 384;
constexpr int kClasses = 3;                       // rows split by r % 3 between fold warps
constexpr int kClassRows = kTileRows / kClasses;  // 128
constexpr int kScratchCols = 48;
constexpr int kCentreCols = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kScratchCol0 = kTileRows;      // scratch buffer b at column 384 + 48 b
constexpr uint32_t kDummyCol0 = kScratchCol0 + 2 * kScratchCols;  // 480..495: fold padding targets
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpGather0 = 2, kWarpFold0 = 6;
constexpr int kGatherWarps = 4, kFoldWarps = 12;
constexpr int kThreads = 32 * (kWarpFold0 + kFoldWarps);  // 576
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kFoldGroup = 16;
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;
constexpr int kMaxSmem = 232448;  // 227 KB opt-in limit per CTA on sm_100

__host__ __device__ constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Shared-memory carve-up, identical on host and device.
template <int BM, int KC>
struct Layout {
    static constexpr int kRowBytes = KC * 2;                      // one gathered row chunk
    static constexpr int kThreadsPerRow = kRowBytes / 16;
    static constexpr int kRowsPerPass = kGatherThreads / kThreadsPerRow;
    static constexpr int kABytes = BM * KC * 2;                   // weight tile per stage
    static constexpr int kAPad = round_up(kABytes, 1024);
    static constexpr int kBPad = round_up(kCentreCols * kRowBytes, 1024);  // up to 128 gathered rows
    static constexpr int kStageBytes = kAPad + kBPad;
    static constexpr uint32_t kSwizzleMask = kRowBytes / 16 - 1;
    static constexpr uint32_t kBLayout = KC == 64 ? 2u : (KC == 32 ? 4u : 6u);  // 128/64/32-byte swizzle
    static constexpr uint32_t kBSbo = 8 * kRowBytes;
    static constexpr int kNAlign = BM == 128 ? 16 : 8;
    static constexpr int kChPerWarp = BM / 4;                     // channels of one TMEM lane quarter

    static constexpr int kNbrBytes = kTileRows * kVol3 * 4;
    static constexpr int kListBytes = kVol3 * kClasses * kClassRows * 2;
    static constexpr int kCntBytes = round_up(kVol3 * kClasses * 4, 16);
    static constexpr int kOutStageBytes = kFoldWarps * 32 * kChPerWarp * 2;
    static constexpr int kMetaBytes = kNbrBytes + kListBytes + kCntBytes + kOutStageBytes + 64 * 8 + 16;

    static int stages() {
        int s = (kMaxSmem - 1024 - kMetaBytes) / kStageBytes;
        return s > 8 ? 8 : s;
    }
    static int smem_bytes(int stages) { return 1024 + stages * kStageBytes + kMetaBytes; }
};

struct Params {
    const int32_t* nbr;  // [n, 27] or null for kernel size 1
    int64_t n;
    int kvol;
    const __nv_bfloat16* x;
    int cin;
    const __nv_bfloat16* bias;
    __nv_bfloat16* out;
    int cout;
    unsigned int* err;
    int stages;
};

// A unit of MMA work: one offset, up to 128 (centre) or 48 (other) columns.
struct Job {
    int k;       // offset (13 = centre for kernel size 3; 0 for kernel size 1)
    int first;   // first row (centre) or first entry of the offset's list (other offsets)
    int n;       // valid columns
    int ncols;   // MMA N (n rounded up)
    bool centre;
};

// Per-offset hit lists.  Offset k's list is the concatenation of three classes
// (rows r with r % 3 == 0, 1, 2), each sorted by row; class c of offset k is
// lists[(3k + c) * 128 + i], i < cnt[3k + c].
__device__ __forceinline__ int list_total(const int* cnt, int k) {
    return cnt[3 * k] + cnt[3 * k + 1] + cnt[3 * k + 2];
}
__device__ __forceinline__ int list_row(const uint16_t* lists, const int* cnt, int k, int e) {
    const int c0 = cnt[3 * k], c1 = cnt[3 * k + 1];
    const int c = (e >= c0) + (e >= c0 + c1);
    const int idx = e - (c >= 1 ? c0 : 0) - (c >= 2 ? c1 : 0);
    return lists[(3 * k + c) * kClassRows + idx];
}

// Enumerates the jobs of a tile in issue order: centre slices, then offsets 0..26
// (skipping the centre) split into kScratchCols-wide parts.  Every role walks the
// same sequence.
struct JobIter {
    const int* cnt;
    int t_eff, kvol, nalign;
    int k, first, total;
    __device__ void start() {
        k = -1;
        first = 0;
    }
    __device__ bool next(Job& j) {
        if (k == -1) {
            if (first < t_eff) {
                j.k = kvol == kVol3 ? kCentre : 0;
                j.first = first;
                j.n = min(kCentreCols, t_eff - first);
                j.ncols = round_up(j.n, nalign);
                j.centre = true;
                first += kCentreCols;
                return true;
            }
            if (kvol != kVol3) return false;
            k = 0;
            first = 0;
            total = list_total(cnt, 0);
        }
        while (k < kVol3) {
            if (k != kCentre && first < total) {
                j.k = k;
                j.first = first;
                j.n = min(kScratchCols, total - first);
                j.ncols = round_up(j.n, nalign);
                j.centre = false;
                first += kScratchCols;
                return true;
            }
            ++k;
            first = 0;
            if (k < kVol3) total = list_total(cnt, k);
        }
        return false;
    }
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
                *abort_flag = 1;
                atomicOr(err, kFwdErrTimeout);
                return false;
            }
        }
    }
}

// Whole-warp wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* err) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag, err) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int BM, int KC>
__global__ void __launch_bounds__(kThreads, 1)
    k_subm_tc(const __grid_constant__ CUtensorMap wmap, const Params p) {
    using L = Layout<BM, KC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.stages;
    uint8_t* stages = smem;
    int32_t* nbr_s = reinterpret_cast<int32_t*>(smem + S * L::kStageBytes);
    uint16_t* lists = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(nbr_s) + L::kNbrBytes);
    int* cnt = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(lists) + L::kListBytes);
    __nv_bfloat16* out_stage = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(cnt) + L::kCntBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(out_stage) + L::kOutStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + S);
    const uint32_t sfull0 = smem_addr(bars + 2 * S), sempty0 = smem_addr(bars + 2 * S + 2);
    const uint32_t accfull = smem_addr(bars + 2 * S + 4), drain = smem_addr(bars + 2 * S + 5);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t)blockIdx.x * kTileRows;
    const int t_eff = (int)min((int64_t)kTileRows, p.n - row0);
    const int cblk = blockIdx.y;
    const int nchunks = p.cin / KC;

    // ---- set-up: barriers, TMEM, neighbour rows of the tile (cp.async, 16 B)
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1 + kGatherThreads);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull0 + 8 * b, 1);
            mbar_init(sempty0 + 8 * b, kFoldWarps);
        }
        mbar_init(accfull, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&wmap);
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (p.kvol == kVol3) {
        // rows row0 .. row0 + t_eff of the map are contiguous: t_eff * 108 bytes,
        // 16-byte aligned because kTileRows * 108 is a multiple of 16.
        const int words = t_eff * kVol3;
        const int vecs = words / 4;
        const int32_t* src = p.nbr + row0 * kVol3;
        const uint32_t dst = smem_addr(nbr_s);
        for (int i = threadIdx.x; i < vecs; i += kThreads) cp_async_16(dst + 16 * i, src + 4 * i, 16);
        for (int i = 4 * vecs + threadIdx.x; i < words; i += kThreads) nbr_s[i] = __ldg(src + i);
        cp_async_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- per-offset, per-class lists of tile rows that have a neighbour
    if (p.kvol == kVol3 && warp >= kWarpGather0) {
        constexpr int kListWarps = kThreads / 32 - kWarpGather0;
        for (int u = warp - kWarpGather0; u < (kVol3 - 1) * kClasses; u += kListWarps) {
            const int ks = u / kClasses, c = u - ks * kClasses;
            const int k = ks < kCentre ? ks : ks + 1;
            int n = 0;
            for (int base = 0; base < kClassRows; base += 32) {
                const int r = c + kClasses * (base + lane);
                const bool hit = r < t_eff && nbr_s[r * kVol3 + k] >= 0;
                const unsigned b = __ballot_sync(0xffffffffu, hit);
                if (hit) lists[(3 * k + c) * kClassRows + n + __popc(b & ((1u << lane) - 1u))] = (uint16_t)r;
                n += __popc(b);
            }
            if (lane == 0) cnt[3 * k + c] = n;
        }
    }
    __syncthreads();

    JobIter it_jobs{cnt, t_eff, p.kvol, L::kNAlign, 0, 0, 0};
    Job job;
    bool aborted = false;

    if (warp == kWarpTma) {
        // ------------------------------------------------ weights via TMA
        if (lane == 0) {
            int it = 0;
            it_jobs.start();
            while (!aborted && it_jobs.next(job)) {
                for (int c = 0; c < nchunks; ++c, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (uint32_t)(it / S) & 1u;
                    if (!wait_bar(empty0 + 8 * s, ph ^ 1u, abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    const uint32_t a_dst = smem_addr(stages + s * L::kStageBytes);
                    mbar_arrive_expect_tx(full0 + 8 * s, L::kABytes);
                    const int y = job.k * p.cin + c * KC;
                    for (int box = 0; box < BM / 64; ++box)
                        tma_load_2d(a_dst + box * KC * 128, &wmap, cblk * BM + box * 64, y, full0 + 8 * s);
                }
            }
            if (aborted) __nanosleep(200000);  // let loads in flight land before the CTA exits
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------ tcgen05.mma issuer
        if (lane == 0) {
            int it = 0, sj = 0;
            it_jobs.start();
            while (!aborted && it_jobs.next(job)) {
                const uint32_t d =
                    tmem + (job.centre ? (uint32_t)job.first : kScratchCol0 + (uint32_t)(sj & 1) * kScratchCols);
                if (!job.centre) {
                    if (!wait_bar(sempty0 + 8 * (sj & 1), ((uint32_t)(sj >> 1) & 1u) ^ 1u, abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                }
                const uint32_t idesc = idesc_bf16(BM, (uint32_t)job.ncols);
                for (int c = 0; c < nchunks; ++c, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (uint32_t)(it / S) & 1u;
                    if (!wait_bar(full0 + 8 * s, ph, abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                    fence_proxy_async_smem();
                    const uint32_t a_base = smem_addr(stages + s * L::kStageBytes);
                    const uint32_t b_base = a_base + L::kAPad;
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk) {
                        const uint64_t adesc = smem_desc(a_base + kk * 2048, KC * 128, 1024, 2);
                        const uint64_t bdesc = smem_desc(b_base + kk * 32, 16, L::kBSbo, L::kBLayout);
                        mma_bf16(d, adesc, bdesc, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(empty0 + 8 * s);
                }
                if (aborted) break;
                if (!job.centre) {
                    mma_commit(sfull0 + 8 * (sj & 1));
                    ++sj;
                }
            }
            if (!aborted) {
                mma_commit(accfull);
            } else {
                mma_commit(drain);  // wait for MMAs in flight before TMEM is freed
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
                }
            }
        }
    } else if (warp < kWarpFold0) {
        // ------------------------------------------------ gather producers
        const int g = threadIdx.x - kWarpGather0 * 32;
        const int q = g % L::kThreadsPerRow;
        const int prow = g / L::kThreadsPerRow;
        int it = 0;
        it_jobs.start();
        while (!aborted && it_jobs.next(job)) {
            for (int c = 0; c < nchunks; ++c, ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                if (!warp_wait_bar(empty0 + 8 * s, ph ^ 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                const uint32_t b_base = smem_addr(stages + s * L::kStageBytes) + L::kAPad;
                const int col_off = c * KC + q * 8;
                for (int pr = prow; pr < job.ncols; pr += L::kRowsPerPass) {
                    const __nv_bfloat16* src = p.x;
                    uint32_t bytes = 0;
                    if (pr < job.n) {
                        int64_t j;
                        if (job.centre) {
                            j = row0 + job.first + pr;
                        } else {
                            const int r = list_row(lists, cnt, job.k, job.first + pr);
                            j = nbr_s[r * kVol3 + job.k];
                        }
                        src = p.x + j * p.cin + col_off;
                        bytes = 16;
                    }
                    const uint32_t lin = (uint32_t)(pr * L::kRowBytes + q * 16);
                    cp_async_16(b_base + (lin ^ (((lin >> 7) & L::kSwizzleMask) << 4)), src, bytes);
                }
                cp_async_mbar_arrive_noinc(full0 + 8 * s);
            }
        }
        cp_async_wait_all();
    } else {
        // ------------------------------------------------ fold scratch -> accumulator, then epilogue
        // Warp (quarter, sub) owns TMEM lanes [32*quarter, +32) and the tile rows
        // r with r % 3 == sub, so every accumulator column is only ever touched by
        // one warp per lane quarter.
        const int quarter = warp & 3;
        const int sub = (warp - kWarpFold0) >> 2;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        int sj = 0;
        it_jobs.start();
        while (!aborted && it_jobs.next(job)) {
            if (job.centre) continue;
            const int b = sj & 1;
            if (!warp_wait_bar(sfull0 + 8 * b, (uint32_t)(sj >> 1) & 1u, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            tc_fence_after();
            const uint32_t scr = tmem + lane_base + kScratchCol0 + (uint32_t)b * kScratchCols;
            const int k = job.k;
            const int cls_start = (sub >= 1 ? cnt[3 * k] : 0) + (sub >= 2 ? cnt[3 * k + 1] : 0);
            const int lo = max(job.first, cls_start);
            const int hi = min(job.first + job.n, cls_start + cnt[3 * k + sub]);
            const uint16_t* lst = lists + (3 * k + sub) * kClassRows;
            bool released = false;
            for (int g0 = lo; g0 < hi; g0 += kFoldGroup) {
                float v[kFoldGroup], a[kFoldGroup];
                uint32_t col[kFoldGroup];
                tmem_ld_x16(scr + (uint32_t)(g0 - job.first), v);
                if (g0 == lo) tmem_wait_st();  // this warp's stores of the previous job have landed
#pragma unroll
                for (int i = 0; i < kFoldGroup; ++i) {
                    const int e = g0 + i;
                    const uint32_t r = lst[min(e, hi - 1) - cls_start];
                    col[i] = tmem + lane_base + (e < hi ? r : kDummyCol0 + (uint32_t)i);
                    tmem_ld_x1(col[i], a[i]);
                }
                tmem_wait_ld();
                if (g0 + kFoldGroup >= hi) {  // last group: the scratch buffer has been read
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty0 + 8 * b);
                    released = true;
                }
#pragma unroll
                for (int i = 0; i < kFoldGroup; ++i) tmem_st_x1(col[i], a[i] + v[i]);
            }
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty0 + 8 * b);
            }
            ++sj;
        }
        tmem_wait_st();
        tc_fence_before();
        named_barrier(1, 32 * kFoldWarps);  // every fold store has landed before any epilogue read
        if (!aborted && warp_wait_bar(accfull, 0, abort_flag, p.err)) {
            tc_fence_after();
            const bool lane_ok = lane < L::kChPerWarp;
            const int ch_base = cblk * BM + quarter * L::kChPerWarp;
            const int ch = ch_base + lane;
            const float bv = (p.bias && lane_ok && ch < p.cout) ? __bfloat162float(p.bias[ch]) : 0.0f;
            __nv_bfloat16* stg = out_stage + (warp - kWarpFold0) * 32 * L::kChPerWarp;
            constexpr int kVecPerRow = L::kChPerWarp * 2 / 16;
            for (int col = 32 * sub; col < t_eff; col += 32 * kClasses) {
                float v[32];
                tmem_ld_x32(tmem + lane_base + (uint32_t)col, v);
                tmem_wait_ld();
                if (lane_ok) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) stg[i * L::kChPerWarp + lane] = __float2bfloat16_rn(v[i] + bv);
                }
                __syncwarp();
                if (ch_base < p.cout) {
                    for (int e = lane; e < 32 * kVecPerRow; e += 32) {
                        const int i = e / kVecPerRow, vq = e % kVecPerRow;
                        if (col + i < t_eff) {
                            const int4 val = *reinterpret_cast<const int4*>(stg + i * L::kChPerWarp + vq * 8);
                            *reinterpret_cast<int4*>(p.out + (row0 + col + i) * p.cout + ch_base + vq * 8) = val;
                        }
                    }
                }
                __syncwarp();
            }
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

template <int BM, int KC>
spconv_status_t launch(const MapData& m, const void* x, int cin, const void* w, const void* bias, void* out,
                       int cout, cudaStream_t stream, cudaError_t* ce) {
    using L = Layout<BM, KC>;
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        *ce = cudaErrorSymbolNotFound;
        return SPCONV_ERR_CUDA;
    }
    const int kvol = m.kernel_size == 3 ? kVol3 : 1;
    // Weights [kvol, cin, cout] viewed as 2-D [kvol*cin rows, cout columns]; a box
    // is 64 output channels (128 B, 128-byte swizzle) by KC input channels.
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)cout, (cuuint64_t)kvol * cin};
    const cuuint64_t strides[1] = {(cuuint64_t)cout * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)KC};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *ce = cudaErrorInvalidValue;
        return SPCONV_ERR_CUDA;
    }
    const int stages = L::stages();
    const int smem = L::smem_bytes(stages);
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [&] {
        attr_err = cudaFuncSetAttribute(k_subm_tc<BM, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err != cudaSuccess) {
        *ce = attr_err;
        return SPCONV_ERR_CUDA;
    }
    Params p;
    p.nbr = m.nbr;
    p.n = m.n;
    p.kvol = kvol;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.cin = cin;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.cout = cout;
    p.err = m.fwd_err;
    p.stages = stages;
    dim3 grid((unsigned)((m.n + kTileRows - 1) / kTileRows), (unsigned)((cout + BM - 1) / BM));
    k_subm_tc<BM, KC><<<grid, kThreads, smem, stream>>>(map, p);
    *ce = cudaGetLastError();
    return *ce == cudaSuccess ? SPCONV_OK : SPCONV_ERR_CUDA;
}

}  // namespace

spconv_status_t launch_forward_tcgen05(const MapData& m, const void* x, int cin, const void* w, const void* bias,
                                       void* out, int cout, cudaStream_t stream, cudaError_t* ce) {
    *ce = cudaSuccess;
    if (cin % 16 != 0 || cout % 64 != 0) return SPCONV_ERR_UNSUPPORTED;
    if (m.n == 0) return SPCONV_OK;
    const bool bm128 = cout % 128 == 0;
    const int kc = cin % 64 == 0 ? 64 : (cin % 32 == 0 ? 32 : 16);
    if (bm128) {
        if (kc == 64) return launch<128, 64>(m, x, cin, w, bias, out, cout, stream, ce);
        if (kc == 32) return launch<128, 32>(m, x, cin, w, bias, out, cout, stream, ce);
        return launch<128, 16>(m, x, cin, w, bias, out, cout, stream, ce);
    }
    if (kc == 64) return launch<64, 64>(m, x, cin, w, bias, out, cout, stream, ce);
    if (kc == 32) return launch<64, 32>(m, x, cin, w, bias, out, cout, stream, ce);
    return launch<64, 16>(m, x, cin, w, bias, out, cout, stream, ce);
}

}  // namespace spconv
