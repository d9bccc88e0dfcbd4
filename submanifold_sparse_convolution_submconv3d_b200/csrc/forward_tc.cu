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
// feature rows are gathered (cp.async, 16 B, zero-filled holes and padding)
// into a swizzled shared-memory tile and multiplied into a scratch buffer, and fold
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

constexpr int kClasses = kTileClasses;           // rows split by r % 3 between fold warps
constexpr int kMaxEntries = (kVol3 - 1) * kTileRows;  // tile metadata entries, worst case
constexpr int kScratchCols = 48;
constexpr int kCentreCols = 48;   // centre jobs: 48-row slices straight into the accumulator
constexpr int kJobRows = 48;      // rows of one job's B tile (centre slice or compacted offset part)
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
    // B tile: kJobRows gathered rows x KC channels, K-major, split into swizzle
    // atoms of up to 64 channels (128 bytes) each: [atom][row][atom row bytes].
    static constexpr int kAtomElems = KC >= 64 ? 64 : KC;
    static constexpr int kAtoms = KC / kAtomElems;
    static constexpr int kAtomRowBytes = kAtomElems * 2;
    static constexpr int kBAtomBytes = kJobRows * kAtomRowBytes;  // 1024-multiple when kAtoms > 1
    static constexpr int kRowBytes = KC * 2;                      // one gathered row chunk
    static constexpr int kThreadsPerRow = kRowBytes / 16;
    static constexpr int kRowsPerPass = kGatherThreads / kThreadsPerRow;
    static constexpr int kChunksPerAtom = kAtomRowBytes / 16;
    static constexpr uint32_t kSwizzleMask = kAtomRowBytes / 16 - 1;
    static constexpr int kABytes = BM * KC * 2;                   // weight tile per stage
    static constexpr int kAPad = round_up(kABytes, 1024);
    static constexpr int kBPad = round_up(kAtoms * kBAtomBytes, 1024);
    static constexpr int kStageBytes = kAPad + kBPad;
    static constexpr uint32_t kBLayout = kAtomRowBytes == 128 ? 2u : (kAtomRowBytes == 64 ? 4u : 6u);
    static constexpr uint32_t kBSbo = 8 * kAtomRowBytes;
    static_assert(kAtoms == 1 || kBAtomBytes % 1024 == 0, "B atoms must keep the swizzle alignment");
    static constexpr int kNAlign = BM == 128 ? 16 : 8;
    static constexpr int kChPerWarp = BM / 4;                     // channels of one TMEM lane quarter

    static constexpr int kEntryJBytes = kMaxEntries * 4;           // neighbour rows of the tile's entries
    static constexpr int kEntryRBytes = kMaxEntries * 2;           // local rows of the tile's entries
    static constexpr int kCntBytes = 2 * kTileCountStride * 4;     // unit counts, then unit starts
    static constexpr int kOutStageBytes = kFoldWarps * 32 * kChPerWarp * 2;
    static constexpr int kMetaBytes = kEntryJBytes + kEntryRBytes + kCntBytes + kOutStageBytes + 64 * 8 + 32;

    static int stages() {
        int s = (kMaxSmem - 1024 - kMetaBytes) / kStageBytes;
        return s > 8 ? 8 : s;
    }
    static int smem_bytes(int stages) { return 1024 + stages * kStageBytes + kMetaBytes; }
};

struct Params {
    const int32_t* tile_counts;  // tile metadata (null for kernel size 1)
    const int64_t* tile_off;
    const uint16_t* pair_r;
    const int32_t* pair_j;
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
    int ks;      // index among the 26 non-centre offsets (other offsets)
    int base;    // flat index of the offset's first entry in the tile metadata
    int first;   // first row (centre) or first entry of the offset's list (other offsets)
    int n;       // valid columns
    int ncols;   // MMA N (n rounded up)
    bool centre;
};

// Per-offset hit lists come from the tile metadata built with the map: offset
// k's entries are the concatenation of its three classes (rows r with r % 3 ==
// 0, 1, 2, each sorted by row), flat indices ustart[3 ks] .. ustart[3 ks + 3).
// Enumerates the jobs of a tile in issue order: centre slices, then the other 26
// offsets, each split into kScratchCols-wide parts.  The order of the 26 offsets
// is rotated per CTA (`rot`) so that CTAs running at the same time request
// different weight tiles instead of all reading the same L2 lines.  Every role
// of a CTA walks the same sequence.
struct JobIter {
    const int* ustart;  // unit starts, ustart[kTileUnits] = number of entries
    int t_eff, kvol, nalign, rot;
    int ki, k, ks, first, total;  // ki: position among the 26 non-centre offsets
    __device__ void start() {
        ki = -1;
        first = 0;
    }
    __device__ void set_offset() {
        ks = (ki + rot) % (kVol3 - 1);
        k = ks < kCentre ? ks : ks + 1;
        total = ustart[3 * ks + 3] - ustart[3 * ks];
        first = 0;
    }
    __device__ bool next(Job& j) {
        if (ki == -1) {
            if (first < t_eff) {
                j.k = kvol == kVol3 ? kCentre : 0;
                j.ks = 0;
                j.base = 0;
                j.first = first;
                j.n = min(kCentreCols, t_eff - first);
                j.ncols = round_up(j.n, nalign);
                j.centre = true;
                first += kCentreCols;
                return true;
            }
            if (kvol != kVol3) return false;
            ki = 0;
            set_offset();
        }
        while (ki < kVol3 - 1) {
            if (first < total) {
                j.k = k;
                j.ks = ks;
                j.base = ustart[3 * ks];
                j.first = first;
                j.n = min(kScratchCols, total - first);
                j.ncols = round_up(j.n, nalign);
                j.centre = false;
                first += kScratchCols;
                return true;
            }
            if (++ki < kVol3 - 1) set_offset();
        }
        return false;
    }
};

// Bounded wait on an mbarrier phase.  `backoff` lets a non-critical waiter sleep
// between polls so that it does not take issue slots from the MMA issuer.
template <bool backoff = false>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (backoff) __nanosleep(64);
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

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Group wait: one thread of the group polls the mbarrier, the whole group then
// meets at a hardware named barrier (blocked warps take no issue slots).  The
// result travels through one of two alternating shared-memory slots.
struct GroupWait {
    int barrier_id, nthreads;
    bool leader;
    volatile int* slots;  // two ints
    int phase;
    __device__ bool operator()(uint32_t bar, uint32_t parity, volatile int* abort_flag, unsigned int* err) {
        volatile int* slot = slots + (phase & 1);
        ++phase;
        if (leader) *slot = wait_bar<true>(bar, parity, abort_flag, err) ? 1 : 0;
        named_barrier(barrier_id, nthreads);
        return *slot != 0;
    }
};

template <int BM, int KC>
__global__ void __launch_bounds__(kThreads, 1)
    k_subm_tc(const __grid_constant__ CUtensorMap wmap, const Params p) {
    using L = Layout<BM, KC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.stages;
    uint8_t* stages = smem;
    int32_t* pj_s = reinterpret_cast<int32_t*>(smem + S * L::kStageBytes);
    uint16_t* pr_s = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(pj_s) + L::kEntryJBytes);
    int* cnt = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(pr_s) + L::kEntryRBytes);
    int* ustart = cnt + kTileCountStride;
    __nv_bfloat16* out_stage = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(cnt) + L::kCntBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(out_stage) + L::kOutStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* wait_slots = abort_flag + 1;  // 2 for the gather group, 2 for the fold group

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
            mbar_init(full0 + 8 * s, 1 + kGatherThreads);  // weight TMA + every gather thread
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
        // The tile's metadata: unit counts (320 B) and entries (local row, neighbour
        // row); every tile's entries start on a multiple of 8, so all copies are
        // 16-byte aligned.
        const int64_t e0 = p.tile_off[blockIdx.x], ne = p.tile_off[blockIdx.x + 1] - e0;
        const uint32_t cnt_dst = smem_addr(cnt), pj_dst = smem_addr(pj_s), pr_dst = smem_addr(pr_s);
        const int32_t* cnt_src = p.tile_counts + (int64_t)blockIdx.x * kTileCountStride;
        for (int i = threadIdx.x; i < kTileCountStride / 4; i += kThreads) cp_async_16(cnt_dst + 16 * i, cnt_src + 4 * i, 16);
        for (int i = threadIdx.x; i < ne / 4; i += kThreads) cp_async_16(pj_dst + 16 * i, p.pair_j + e0 + 4 * i, 16);
        for (int i = threadIdx.x; i < ne / 8; i += kThreads) cp_async_16(pr_dst + 16 * i, p.pair_r + e0 + 8 * i, 16);
        cp_async_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- flat start of every (offset, class) unit
    if (p.kvol == kVol3 && warp == 0) {
        int run = 0;
        for (int base = 0; base < kTileUnits; base += 32) {
            const int u = base + lane;
            const int c = u < kTileUnits ? cnt[u] : 0;
            int incl = c;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            if (u < kTileUnits) ustart[u] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) ustart[kTileUnits] = run;
    }
    __syncthreads();

    JobIter it_jobs{ustart, t_eff, p.kvol, L::kNAlign, (int)((blockIdx.x * 11u + blockIdx.y * 5u) % (kVol3 - 1)),
                    0, 0, 0, 0, 0};
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
                    if (!wait_bar<true>(empty0 + 8 * s, ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag, p.err)) {
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
                }
                const uint32_t idesc = idesc_bf16(BM, (uint32_t)job.ncols);
                for (int c = 0; c < nchunks; ++c, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (uint32_t)(it / S) & 1u;
                    if (!wait_bar(full0 + 8 * s, ph, abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    const uint32_t a_base = smem_addr(stages + s * L::kStageBytes);
                    const uint32_t b_base = a_base + L::kAPad;
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk) {
                        const uint64_t adesc = smem_desc(a_base + kk * 2048, KC * 128, 1024, 2);
                        constexpr int kStepsPerAtom = L::kAtomElems / 16;
                        const uint64_t bdesc =
                            smem_desc(b_base + (kk / kStepsPerAtom) * L::kBAtomBytes + (kk % kStepsPerAtom) * 32, 16,
                                      L::kBSbo, L::kBLayout);
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
        // The four warps fill every stage together.  Per job: resolve this
        // thread's source rows once (independent shared-memory lookups), then
        // issue the 16-byte copies of every input-channel chunk.  Each thread
        // arrives on the stage barrier when its own copies land
        // (cp.async.mbarrier.arrive.noinc), so no producer ever waits for data.
        constexpr int kMaxPass = (kJobRows + L::kRowsPerPass - 1) / L::kRowsPerPass;
        const int g = threadIdx.x - kWarpGather0 * 32;
        GroupWait gwait{3, kGatherThreads, g == 0, wait_slots, 0};
        const int q = g % L::kThreadsPerRow;
        const int prow = g / L::kThreadsPerRow;
        const int atom = q / L::kChunksPerAtom, qa = q % L::kChunksPerAtom;
        int it = 0;
        it_jobs.start();
        while (!aborted && it_jobs.next(job)) {
            int64_t src_row[kMaxPass];
            uint32_t dst_off[kMaxPass];
#pragma unroll
            for (int ps = 0; ps < kMaxPass; ++ps) {
                const int pr = prow + ps * L::kRowsPerPass;
                src_row[ps] = -1;
                if (pr < job.n) src_row[ps] = job.centre ? row0 + job.first + pr : (int64_t)pj_s[job.base + job.first + pr];
                const uint32_t lin = (uint32_t)(pr * L::kAtomRowBytes + qa * 16);
                dst_off[ps] = (uint32_t)(atom * L::kBAtomBytes) + (lin ^ (((lin >> 7) & L::kSwizzleMask) << 4));
            }
            for (int c = 0; c < nchunks; ++c, ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                if (!gwait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                const uint32_t b_base = smem_addr(stages + s * L::kStageBytes) + L::kAPad;
#pragma unroll
                for (int ps = 0; ps < kMaxPass; ++ps) {
                    const int pr = prow + ps * L::kRowsPerPass;
                    if (pr < job.ncols) {
                        const bool hit = src_row[ps] >= 0;
                        cp_async_16(b_base + dst_off[ps], p.x + (hit ? src_row[ps] : 0) * p.cin + c * KC + q * 8,
                                    hit ? 16u : 0u);
                    }
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
        GroupWait fwait{2, 32 * kFoldWarps, threadIdx.x == kWarpFold0 * 32, wait_slots + 2, 0};
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        int sj = 0;
        it_jobs.start();
        while (!aborted && it_jobs.next(job)) {
            if (job.centre) continue;
            const int b = sj & 1;
            if (!fwait(sfull0 + 8 * b, (uint32_t)(sj >> 1) & 1u, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            const uint32_t scr = tmem + lane_base + kScratchCol0 + (uint32_t)b * kScratchCols;
            // this warp's class of the job's offset: flat entries [cls_lo, cls_hi)
            const int cls_lo = ustart[3 * job.ks + sub] - job.base, cls_hi = ustart[3 * job.ks + sub + 1] - job.base;
            const int lo = max(job.first, cls_lo);
            const int hi = min(job.first + job.n, cls_hi);
            const uint16_t* lst = pr_s + job.base;
            // 1) read this warp's scratch columns with wide loads and hand the
            //    buffer back to the MMA issuer at once;
            float v[kScratchCols];
            const int ng = (hi - lo + kFoldGroup - 1) / kFoldGroup;  // <= 3
            if (ng > 0) tmem_ld_x16(scr + (uint32_t)(lo - job.first), v);
            if (ng > 1) tmem_ld_x16(scr + (uint32_t)(lo - job.first + kFoldGroup), v + kFoldGroup);
            if (ng > 2) tmem_ld_x16(scr + (uint32_t)(lo - job.first + 2 * kFoldGroup), v + 2 * kFoldGroup);
            tmem_wait_ld();  // the scratch values are in registers
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty0 + 8 * b);
            // 2) then add them into the accumulator columns of their rows.
            if (ng > 0) tmem_wait_st();  // this warp's stores of the previous job have landed
#pragma unroll
            for (int gi = 0; gi < kScratchCols / kFoldGroup; ++gi) {
                if (gi < ng) {
                    const int g0 = lo + gi * kFoldGroup;
                    float a[kFoldGroup];
                    uint32_t col[kFoldGroup];
#pragma unroll
                    for (int i = 0; i < kFoldGroup; ++i) {
                        const int e = g0 + i;
                        const uint32_t r = lst[min(e, hi - 1)];
                        col[i] = tmem + lane_base + (e < hi ? r : kDummyCol0 + (uint32_t)i);
                        tmem_ld_x1(col[i], a[i]);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < kFoldGroup; ++i) tmem_st_x1(col[i], a[i] + v[gi * kFoldGroup + i]);
                }
            }
            ++sj;
        }
        tmem_wait_st();
        tc_fence_before();
        named_barrier(1, 32 * kFoldWarps);  // every fold store has landed before any epilogue read
        if (!aborted && fwait(accfull, 0, abort_flag, p.err)) {
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
    p.tile_counts = m.tile_counts;
    p.tile_off = m.tile_off;
    p.pair_r = m.pair_r;
    p.pair_j = m.pair_j;
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
    const int kc = cin % 128 == 0 ? 128 : (cin % 64 == 0 ? 64 : (cin % 32 == 0 ? 32 : 16));
    if (bm128) {
        if (kc == 128) return launch<128, 128>(m, x, cin, w, bias, out, cout, stream, ce);
        if (kc == 64) return launch<128, 64>(m, x, cin, w, bias, out, cout, stream, ce);
        if (kc == 32) return launch<128, 32>(m, x, cin, w, bias, out, cout, stream, ce);
        return launch<128, 16>(m, x, cin, w, bias, out, cout, stream, ce);
    }
    if (kc == 128) return launch<64, 128>(m, x, cin, w, bias, out, cout, stream, ce);
    if (kc == 64) return launch<64, 64>(m, x, cin, w, bias, out, cout, stream, ce);
    if (kc == 32) return launch<64, 32>(m, x, cin, w, bias, out, cout, stream, ce);
    return launch<64, 16>(m, x, cin, w, bias, out, cout, stream, ce);
}

}  // namespace spconv
