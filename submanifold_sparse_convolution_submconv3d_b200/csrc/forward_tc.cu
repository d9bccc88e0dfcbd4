// Fused gather -> tcgen05 GEMM -> single-write store, bf16 in, fp32 accumulate.
//
// The pages fuse the 27 per-offset taps into one [N, 27*Cin] x [27*Cin, Cout]
// matmul over a cached device index (lato.2_mrp_mlx README, "Fleet benchmark"
// and the optimisation table after it).  This kernel computes the same sum, laid
// out for sm_100a:
//
//   D^T[Cout_blk, rows] = sum_k W_k^T[Cout_blk, Cin] . X_k^T[Cin, rows]
//
// One CTA owns a tile of consecutive output rows (at most kTileRows, chosen per
// map so that the tiles fill whole waves of SMs) and one block of 64 or 128
// output channels.  Tensor memory (TMEM, 128 lanes x 512 fp32 columns) holds
//   * the accumulator: lane = output channel, column = output row of the tile;
//   * two scratch buffers of kJobRows columns and 16 dummy columns.
// Work is cut into jobs listed once per tile in shared memory.  First the centre
// offset (every row is its own neighbour): its feature rows are contiguous, so
// they arrive by a tiled TMA load, BM rows per job, and the products go straight
// into the accumulator; with kernel size 1 this is the whole layer, a plain
// TMA-fed tensor-core GEMM.  Then, for every other offset, the compacted list of
// tile rows that have a neighbour there, in parts of at most kJobRows entries:
// their neighbour feature rows are gathered (cp.async, 16 B, zero-filled padding)
// into a swizzled shared-memory tile and multiplied into a scratch buffer, and
// fold warps add each scratch column into the accumulator column of its row
// (tcgen05.ld / tcgen05.st, no atomics).  W_k arrives by TMA once per offset
// (once per job and channel chunk when Cin spans several chunks, and once per
// centre job).  At the end each output row is written exactly once, with bias,
// rounded to bf16.
//
// Warp roles (608 threads):
//   warps 1, 18 TMEM allocator (warp 1) and the two tcgen05.mma issuers, which
//               take alternate jobs
//   warp 5      TMA producer of weight tiles (A operand), a ring of 2-6 slots
//   warps 0, 2-4  gather producers (B operand): gather warp g fills the offset
//               jobs ncj + q (ncj centre jobs first) with q % 4 == g into its own
//               ring of slots, in order, so each ring is filled and drained
//               strictly in sequence
//   warps 6-17  scratch -> accumulator fold, then the epilogue: three warps per
//               TMEM lane quarter, each owning the tile rows of one residue mod 3,
//               so no accumulator column is touched by two warps of a quarter.
//               Narrow TMEM accesses go in batches of kNarrowGroup loads, one
//               wait, then the stores, without per-element branches; padding
//               entries go to dedicated dummy columns.
// Waiting threads are suspended on their mbarrier (try_wait with a time hint)
// and take no issue slots.  Every wait is bounded: after kWaitTimeoutNs the
// kernel records kFwdErrTimeout in the map's error word, stops issuing work,
// lets copies in flight land, frees its TMEM and returns.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"

namespace spconv {
namespace {

using namespace sm100;

constexpr int kClasses = kTileClasses;                   // rows split by r % 3 between fold warps
constexpr int kJobRows = 48;                             // columns of one job (MMA N <= 48)
constexpr int kMaxJobs = (kTileRows + kJobRows - 1) / kJobRows * kVol3;  // at most 8 jobs per offset
constexpr int kScratchBufs = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kScratchCol0 = kTileRows;             // scratch buffer b at column 384 + 48 b
constexpr uint32_t kDummyCol0 = kScratchCol0 + kScratchBufs * kJobRows;  // 480..495: fold padding targets
static_assert(kDummyCol0 + 16 <= kTmemCols, "accumulator, scratch buffers and dummy columns must fit TMEM");
// Warp w runs on sub-partition w % 4, and a fold warp must sit on the
// sub-partition of its TMEM lane quarter.  The first MMA issuer's sub-partition
// (1) therefore hosts, besides three fold warps, only the light weight producer;
// the four gather warps (0, 2, 3, 4) and the second issuer (18) go to the others.
constexpr int kWarpMma = 1, kWarpTma = 5, kWarpFold0 = 6, kWarpMma2 = 18;
constexpr int kGatherWarps = 4, kFoldWarps = 12;
constexpr int kThreads = 32 * (kWarpFold0 + kFoldWarps + 1);  // 608
constexpr int kFoldGroup = 16;    // scratch columns per wide TMEM load
constexpr int kNarrowGroup = 8;   // accumulator columns per batch of narrow loads, then stores
constexpr int kMaxASlots = 6;                             // weight ring slots
constexpr int kMaxBSlots = 8;                             // gather ring slots per gather warp
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;
constexpr uint32_t kSuspendHintNs = 20000;
constexpr int kMaxSmem = 232448;  // 227 KB opt-in limit per CTA on sm_100

__host__ __device__ constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Job record (int4): x = k | ks << 8 | centre << 16 | gather slot << 17 | slot
// phase << 20 (slot and phase of the job's first channel chunk in its gather
// warp's ring), y = first local row (centre) or first flat entry of the tile's
// lists, z = valid columns n, w = MMA N.
__device__ __forceinline__ int job_k(const int4& j) { return j.x & 0xFF; }
__device__ __forceinline__ int job_ks(const int4& j) { return (j.x >> 8) & 0xFF; }
__device__ __forceinline__ bool job_centre(const int4& j) { return (j.x >> 16) & 1; }
__device__ __forceinline__ int job_bslot(const int4& j) { return (j.x >> 17) & 7; }
__device__ __forceinline__ uint32_t job_bphase(const int4& j) { return (uint32_t)(j.x >> 20) & 1u; }

// Shared-memory carve-up, identical on host and device:
//   [weight ring][gather rings][job table][unit counts, unit starts]
//   [neighbour rows][local rows][mbarriers][misc words]
// The epilogue's staging buffer reuses the start of the rings once every MMA is done.
template <int BM, int KC>
struct Layout {
    // B tile: kJobRows gathered rows x KC channels, K-major, split into swizzle
    // atoms of up to 64 channels (128 bytes) each: [atom][row][atom row bytes].
    static constexpr int kAtomElems = KC >= 64 ? 64 : KC;
    static constexpr int kAtoms = KC / kAtomElems;
    static constexpr int kAtomRowBytes = kAtomElems * 2;
    static constexpr int kBAtomBytes = kJobRows * kAtomRowBytes;  // 1024-multiple when kAtoms > 1
    static constexpr int kThreadsPerRow = KC * 2 / 16;            // 16-byte chunks of one row chunk
    static constexpr int kWarpRows = 32 / kThreadsPerRow;         // rows one warp instruction covers
    static constexpr int kPasses = kJobRows / kWarpRows;
    static constexpr int kGatherBatch = kPasses % 8 == 0 ? 8 : (kPasses % 6 == 0 ? 6 : kPasses);
    static_assert(kPasses % kGatherBatch == 0, "gather batches must cover every pass");
    static constexpr int kChunksPerAtom = kAtomRowBytes / 16;
    static constexpr uint32_t kSwizzleMask = kAtomRowBytes / 16 - 1;
    static constexpr int kABytes = BM * KC * 2;                   // weight tile per slot
    static constexpr int kAPad = round_up(kABytes, 1024);
    static constexpr int kBPad = round_up(kAtoms * kBAtomBytes, 1024);
    static constexpr uint32_t kBLayout = kAtomRowBytes == 128 ? 2u : (kAtomRowBytes == 64 ? 4u : 6u);
    static constexpr uint32_t kBSbo = 8 * kAtomRowBytes;
    static_assert(kAtoms == 1 || kBAtomBytes % 1024 == 0, "B atoms must keep the swizzle alignment");
    static_assert(kJobRows % kWarpRows == 0, "a job must split into whole warp passes");
    static constexpr int kNAlign = BM == 128 ? 16 : 8;
    static constexpr int kChPerWarp = BM / 4;                     // channels of one TMEM lane quarter
    static constexpr int kOutStageBytes = kFoldWarps * 32 * kChPerWarp * 2;
    static constexpr int kFixedMeta = kMaxJobs * 16 + 2 * kTileCountStride * 4;

    __host__ __device__ static int ring_bytes(int sa, int sb) { return sa * kAPad + kGatherWarps * sb * kBPad; }
    __host__ __device__ static int num_bars(int sa, int sb) { return 2 * sa + 2 * kGatherWarps * sb + 2 * kScratchBufs + 4; }
    __host__ __device__ static int smem_bytes(int cap, int sa, int sb) {
        return 1024 + ring_bytes(sa, sb) + kFixedMeta + cap * 4 + round_up(cap * 2, 16) + num_bars(sa, sb) * 8 + 16;
    }
    static bool fits(int cap, int sa, int sb) { return smem_bytes(cap, sa, sb) <= kMaxSmem; }
    // Ring depths for a tile entry capacity `cap`.  Gather depth matters more than
    // weight depth (measured): keep three weight slots (two if nothing else fits;
    // a centre job holds two at once), give the room to gather slots, then any
    // room left back to weight slots.  The rings must also hold the epilogue's
    // staging buffer.  {0, 0} if nothing fits.
    static void depths(int cap, int* sa, int* sb) {
        *sa = 0;
        *sb = 0;
        for (int a_min = 3; a_min >= 2; --a_min) {
            if (!fits(cap, a_min, 1)) continue;
            int b = 1;
            while (b < kMaxBSlots && fits(cap, a_min, b + 1)) ++b;
            int a = a_min;
            while (a < kMaxASlots && fits(cap, a + 1, b)) ++a;
            if (ring_bytes(a, b) < kOutStageBytes) continue;
            *sa = a;
            *sb = b;
            return;
        }
    }
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
    int tile_rows;  // rows per tile (<= kTileRows)
    int sa;   // weight ring slots
    int sb;   // gather slots per gather warp
    int cap;  // entry capacity of the shared-memory lists (largest tile's entries)
};

// Bounded wait on an mbarrier phase; the thread sleeps inside try_wait.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err) {
    if (mbar_try_wait_hint(bar, parity, kSuspendHintNs)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_hint(bar, parity, kSuspendHintNs)) return true;
        if ((i & 15u) != 0) continue;  // the timer and the abort flag every few wake-ups
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            atomicOr(err, kFwdErrTimeout);
            return false;
        }
    }
}

// Lane 0 waits, the warp learns the outcome.
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* err) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag, err) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int BM, int KC>
__global__ void __launch_bounds__(kThreads, 1)
    k_subm_tc(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, const Params p) {
    using L = Layout<BM, KC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int SA = p.sa, SB = p.sb;
    uint8_t* a_ring = smem;
    uint8_t* b_ring = smem + SA * L::kAPad;
    int4* jobs = reinterpret_cast<int4*>(smem + L::ring_bytes(SA, SB));
    int* cnt = reinterpret_cast<int*>(jobs + kMaxJobs);
    int* ustart = cnt + kTileCountStride;
    int32_t* pj_s = reinterpret_cast<int32_t*>(ustart + kTileCountStride);
    uint16_t* pr_s = reinterpret_cast<uint16_t*>(pj_s + p.cap);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(pr_s) + round_up(p.cap * 2, 16));
    int* misc = reinterpret_cast<int*>(bars + L::num_bars(SA, SB));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_flag = misc + 1;
    __nv_bfloat16* out_stage = reinterpret_cast<__nv_bfloat16*>(smem);

    const uint32_t fullA0 = smem_addr(bars), emptyA0 = fullA0 + 8 * SA;
    const uint32_t fullB0 = emptyA0 + 8 * SA, emptyB0 = fullB0 + 8 * kGatherWarps * SB;
    const uint32_t sfull0 = emptyB0 + 8 * kGatherWarps * SB, sempty0 = sfull0 + 8 * kScratchBufs;
    const uint32_t accfull = sempty0 + 8 * kScratchBufs, drain0 = accfull + 8;  // drain0, drain1: one per issuer
    const uint32_t centre_done = drain0 + 16;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t)blockIdx.x * p.tile_rows;
    const int t_eff = (int)min((int64_t)p.tile_rows, p.n - row0);
    const int cblk = blockIdx.y;
    const int nchunks = p.cin / KC;

    // ---- set-up: barriers, TMEM, the tile's lists (cp.async, 16 B).  The weight
    // producer initialises the barriers and at once issues the first two ring uses,
    // which every tile has (centre weights and the first BM centre rows, first
    // channel chunk), so their latency overlaps the set-up and the job table.
    if (threadIdx.x == kWarpTma * 32) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(fullA0 + 8 * s, 1);
            mbar_init(emptyA0 + 8 * s, 2);  // both issuers release every weight-ring use
        }
        for (int s = 0; s < kGatherWarps * SB; ++s) {
            mbar_init(fullB0 + 8 * s, 32);  // the 32 lanes of the filling gather warp
            mbar_init(emptyB0 + 8 * s, 1);
        }
        for (int b = 0; b < kScratchBufs; ++b) {
            mbar_init(sfull0 + 8 * b, 1);
            mbar_init(sempty0 + 8 * b, kFoldWarps);
        }
        mbar_init(accfull, 2);
        mbar_init(drain0, 1);
        mbar_init(drain0 + 8, 1);
        mbar_init(centre_done, 2);
        *abort_flag = 0;
        fence_mbar_init();
        const int kc = p.kvol == kVol3 ? kCentre : 0;
        mbar_arrive_expect_tx(fullA0, L::kABytes);
        for (int box = 0; box < BM / 64; ++box)
            tma_load_2d(smem_addr(a_ring) + box * KC * 128, &wmap, cblk * BM + box * 64, kc * p.cin, fullA0);
        mbar_arrive_expect_tx(fullA0 + 8, L::kABytes);
        for (int a = 0; a < L::kAtoms; ++a)
            tma_load_2d(smem_addr(a_ring + L::kAPad) + a * BM * L::kAtomRowBytes, &xmap, a * L::kAtomElems, (int)row0,
                        fullA0 + 8);
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (p.kvol == kVol3) {
        // Unit counts (320 B) and entries (neighbour row, local row); every tile's
        // entries start on a multiple of 8, so all copies are 16-byte aligned.
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

    // ---- job table (warp 0): centre slices of BM rows, then every other
    // offset's list in 48-entry parts.  The order of the 26 offsets is rotated per
    // CTA so that CTAs running at the same time request different weight tiles.
    if (warp == 0) {
        const int kc = p.kvol == kVol3 ? kCentre : 0;
        const int ncj = (t_eff + BM - 1) / BM;
        for (int j = lane; j < ncj; j += 32) {
            const int n = min(BM, t_eff - j * BM);
            jobs[j] = make_int4(kc | (1 << 16), j * BM, n, round_up(n, L::kNAlign));
        }
        int njobs = ncj;
        if (p.kvol == kVol3) {
            int run = 0;  // flat start of every (offset, class) unit
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
            __syncwarp();
            const int rot = (int)((blockIdx.x * 11u + blockIdx.y * 5u) % (kVol3 - 1));
            int ks = 0, e0 = 0, tot = 0, nj = 0;
            if (lane < kVol3 - 1) {
                ks = (lane + rot) % (kVol3 - 1);
                e0 = ustart[3 * ks];
                tot = ustart[3 * ks + 3] - e0;
                nj = (tot + kJobRows - 1) / kJobRows;
            }
            int incl = nj;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            const int start = ncj + incl - nj;
            const int k = ks < kCentre ? ks : ks + 1;
            for (int q = 0; q < nj; ++q) {
                const int n = min(kJobRows, tot - q * kJobRows);
                jobs[start + q] = make_int4(k | (ks << 8), e0 + q * kJobRows, n, round_up(n, L::kNAlign));
            }
            njobs = ncj + __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncwarp();
        // first gather slot and phase of every offset job: job ncj + q is the
        // (q / 4)-th of gather warp q % 4, whose ring has advanced by nchunks per
        // earlier job
        for (int j = ncj + lane; j < njobs; j += 32) {
            const int u0 = ((j - ncj) / kGatherWarps) * nchunks;
            jobs[j].x |= ((u0 % SB) << 17) | (((u0 / SB) & 1) << 20);
        }
        if (lane == 0) {
            misc[2] = njobs;
            misc[3] = ncj;
        }
    }
    __syncthreads();
    const int njobs = misc[2], ncj = misc[3];
    bool aborted = false;

    if (warp == kWarpTma) {
        // ------------------------------------------------ weights (and centre rows) via TMA
        // Ring uses, in the issuer's order: per centre job and channel chunk the
        // centre weights then the job's BM feature rows; per offset (per job and
        // chunk when Cin spans several chunks) the offset's weights.
        if (lane == 0) {
            int s = 2 % SA, prev_k = -1;  // the first two uses were issued during set-up
            uint32_t ph = (uint32_t)(2 / SA) & 1u;
            for (int j = 0; j < njobs && !aborted; ++j) {
                const int4 jb = jobs[j];
                const int k = job_k(jb);
                const bool centre = job_centre(jb);
                if (!centre && nchunks == 1 && k == prev_k) continue;  // same offset: the loaded tile serves
                prev_k = k;
                for (int c = 0; c < nchunks && !aborted; ++c) {
                    if (j == 0 && c == 0) continue;  // issued during set-up
                    for (int part = 0; part < (centre ? 2 : 1); ++part) {
                        if (!wait_bar(emptyA0 + 8 * s, ph ^ 1u, abort_flag, p.err)) {
                            aborted = true;
                            break;
                        }
                        const uint32_t dst = smem_addr(a_ring + s * L::kAPad);
                        mbar_arrive_expect_tx(fullA0 + 8 * s, L::kABytes);
                        if (part == 0) {
                            const int y = k * p.cin + c * KC;
                            for (int box = 0; box < BM / 64; ++box)
                                tma_load_2d(dst + box * KC * 128, &wmap, cblk * BM + box * 64, y, fullA0 + 8 * s);
                        } else {
                            // BM feature rows [row0 + first, +BM) x KC channels, K-major in
                            // swizzle atoms (rows past the last voxel read as zeros)
                            for (int a = 0; a < L::kAtoms; ++a)
                                tma_load_2d(dst + a * BM * L::kAtomRowBytes, &xmap, c * KC + a * L::kAtomElems,
                                            (int)row0 + jb.y, fullA0 + 8 * s);
                        }
                        if (++s == SA) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                }
            }
            if (aborted) __nanosleep(200000);  // let loads in flight land before the CTA exits
        }
    } else if (warp == kWarpMma || warp == kWarpMma2) {
        // ------------------------------------------------ tcgen05.mma issuers
        // Two issuer threads take alternate jobs (issuer me owns the jobs j with
        // j % 2 == me), so one's bookkeeping and waits overlap the other's MMAs.
        //  * Weight ring: both walk every ring use in order, wait for it to fill and
        //    commit its release once (the slot's empty barrier counts two), so no
        //    issuer can run a ring length ahead of the other.
        //  * Gather rings: offset job ncj + q comes from gather warp q % 4, and
        //    (ncj + q) % 2 = me keeps each gather warp's jobs with one issuer.
        //  * Scratch buffers: offset job ncj + q uses buffer q % 2, so each issuer
        //    owns one buffer and uses it in order.
        //  * The fold starts after both issuers' centre MMAs (centre_done).
        if (lane == 0) {
            const int me = warp == kWarpMma ? 0 : 1;
            const int own_b = (me + ncj) & 1;  // this issuer's scratch buffer
            uint32_t own_ph = 1u;              // parity of its previous use
            int as = SA - 1, prev_k = -1;      // weight slot in use and its phase
            uint32_t aph = 1u;
            int4 jb = njobs > 0 ? jobs[0] : make_int4(0, 0, 0, 0);
            for (int j = 0; j < njobs && !aborted; ++j) {
                const int4 jn = j + 1 < njobs ? jobs[j + 1] : make_int4(-1, 0, 0, 0);  // prefetch
                const int k = job_k(jb);
                const bool centre = job_centre(jb);
                const bool mine = (j & 1) == me;
                const bool new_k = k != prev_k;
                prev_k = k;
                const bool last_of_k = j + 1 == njobs || job_k(jn) != k;
                uint32_t d = tmem + (uint32_t)jb.y;
                if (mine && !centre) {
                    own_ph ^= 1u;
                    d = tmem + kScratchCol0 + (uint32_t)own_b * kJobRows;
                    if (!wait_bar(sempty0 + 8 * own_b, own_ph ^ 1u, abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                }
                const uint32_t idesc = idesc_bf16(BM, (uint32_t)jb.w);
                if (centre) {
                    // weights and feature rows both come through the TMA ring
                    for (int c = 0; c < nchunks; ++c) {
                        int ws = 0;
                        for (int part = 0; part < 2; ++part) {
                            if (++as == SA) {
                                as = 0;
                                aph ^= 1u;
                            }
                            if (part == 0) ws = as;
                            if (!wait_bar(fullA0 + 8 * as, aph, abort_flag, p.err)) {
                                aborted = true;
                                break;
                            }
                        }
                        if (aborted) break;
                        if (mine) {
                            const uint32_t a_base = smem_addr(a_ring + ws * L::kAPad);
                            const uint32_t x_base = smem_addr(a_ring + as * L::kAPad);
#pragma unroll
                            for (int kk = 0; kk < KC / 16; ++kk) {
                                const uint64_t adesc = smem_desc(a_base + kk * 2048, KC * 128, 1024, 2);
                                constexpr int kStepsPerAtom = L::kAtomElems / 16;
                                const uint64_t bdesc = smem_desc(
                                    x_base + (kk / kStepsPerAtom) * (BM * L::kAtomRowBytes) + (kk % kStepsPerAtom) * 32,
                                    16, L::kBSbo, L::kBLayout);
                                mma_bf16(d, adesc, bdesc, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        mma_commit(emptyA0 + 8 * ws);
                        mma_commit(emptyA0 + 8 * as);
                    }
                    if (aborted) break;
                    if (j == ncj - 1) mma_commit(centre_done);
                    jb = jn;
                    continue;
                }
                const int gw = (j - ncj) & (kGatherWarps - 1);
                int bs = job_bslot(jb);
                uint32_t bph = job_bphase(jb);
                for (int c = 0; c < nchunks; ++c) {
                    if (nchunks > 1 || (c == 0 && new_k)) {
                        if (++as == SA) {
                            as = 0;
                            aph ^= 1u;
                        }
                        if (!wait_bar(fullA0 + 8 * as, aph, abort_flag, p.err)) {
                            aborted = true;
                            break;
                        }
                    }
                    if (mine) {
                        const int bslot = gw * SB + bs;
                        if (!wait_bar(fullB0 + 8 * bslot, bph, abort_flag, p.err)) {
                            aborted = true;
                            break;
                        }
                        // the B tile was written by cp.async (generic proxy); the MMA reads it
                        // through the async proxy
                        fence_proxy_async_smem();
                        const uint32_t a_base = smem_addr(a_ring + as * L::kAPad);
                        const uint32_t b_base = smem_addr(b_ring + bslot * L::kBPad);
#pragma unroll
                        for (int kk = 0; kk < KC / 16; ++kk) {
                            const uint64_t adesc = smem_desc(a_base + kk * 2048, KC * 128, 1024, 2);
                            constexpr int kStepsPerAtom = L::kAtomElems / 16;
                            const uint64_t bdesc =
                                smem_desc(b_base + (kk / kStepsPerAtom) * L::kBAtomBytes + (kk % kStepsPerAtom) * 32,
                                          16, L::kBSbo, L::kBLayout);
                            mma_bf16(d, adesc, bdesc, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(emptyB0 + 8 * bslot);
                        if (++bs == SB) {
                            bs = 0;
                            bph ^= 1u;
                        }
                    }
                    if (nchunks > 1 || last_of_k) mma_commit(emptyA0 + 8 * as);
                }
                if (aborted) break;
                if (mine) mma_commit(sfull0 + 8 * own_b);
                jb = jn;
            }
            if (!aborted) {
                mma_commit(accfull);
            } else {
                const uint32_t drain = drain0 + 8 * me;
                mma_commit(drain);  // wait for this issuer's MMAs in flight before TMEM is freed
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
                }
            }
        }
    } else if (warp < kWarpFold0) {
        // ------------------------------------------------ gather producers
        // Lane l copies 16-byte chunk l % kThreadsPerRow of rows
        // l / kThreadsPerRow + kWarpRows * pass, looking the source rows up in
        // batches.  Each lane arrives on the slot's barrier when its own copies land
        // (cp.async.mbarrier.arrive.noinc), so no producer ever waits for data.
        const int gw = warp == 0 ? 0 : warp - 1;
        const int q = lane % L::kThreadsPerRow;
        const int prow = lane / L::kThreadsPerRow;
        const int atom = q / L::kChunksPerAtom, qa = q % L::kChunksPerAtom;
        int s = 0;
        uint32_t ph = 0;
        for (int j = ncj + gw; j < njobs && !aborted; j += kGatherWarps) {
            const int4 jb = jobs[j];
            const int n = jb.z, ncols = jb.w;
            for (int c = 0; c < nchunks; ++c) {
                const int slot = gw * SB + s;
                if (!warp_wait_bar(emptyB0 + 8 * slot, ph ^ 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                const uint32_t b_base = smem_addr(b_ring + slot * L::kBPad) + (uint32_t)(atom * L::kBAtomBytes);
                const __nv_bfloat16* xc = p.x + c * KC + q * 8;
                // batches of row lookups then copies, in a rolled loop: a fully unrolled
                // job (24 passes at 128 channels) measured 6 % slower overall
#pragma unroll 1
                for (int h = 0; h < L::kPasses / L::kGatherBatch; ++h) {
                    int src[L::kGatherBatch];
#pragma unroll
                    for (int i = 0; i < L::kGatherBatch; ++i) {
                        const int pr = prow + (h * L::kGatherBatch + i) * L::kWarpRows;
                        src[i] = pr < n ? pj_s[jb.y + pr] : -1;
                    }
#pragma unroll
                    for (int i = 0; i < L::kGatherBatch; ++i) {
                        const int pr = prow + (h * L::kGatherBatch + i) * L::kWarpRows;
                        if (pr < ncols) {
                            const uint32_t lin = (uint32_t)(pr * L::kAtomRowBytes + qa * 16);
                            const bool hit = src[i] >= 0;
                            cp_async_16(b_base + (lin ^ (((lin >> 7) & L::kSwizzleMask) << 4)),
                                        xc + (int64_t)(hit ? src[i] : 0) * p.cin, hit ? 16u : 0u);
                        }
                    }
                }
                cp_async_mbar_arrive_noinc(fullB0 + 8 * slot);
                if (++s == SB) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        cp_async_wait_all();
    } else if (warp < kWarpFold0 + kFoldWarps) {
        // ------------------------------------------------ fold scratch -> accumulator, then epilogue
        // Warp (quarter, sub) owns TMEM lanes [32*quarter, +32) and the tile rows
        // r with r % 3 == sub, so every accumulator column is only ever touched by
        // one warp per lane quarter.
        const int quarter = warp & 3;
        const int sub = (warp - kWarpFold0) >> 2;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        int b = kScratchBufs - 1;  // scratch buffer of the current offset job and its phase
        uint32_t sph = 1u;
        // both issuers' centre MMAs write accumulator columns: they complete first
        if (warp_wait_bar(centre_done, 0, abort_flag, p.err))
            tc_fence_after();
        else
            aborted = true;
        for (int j = 0; j < njobs && !aborted; ++j) {
            const int4 jb = jobs[j];
            if (job_centre(jb)) continue;
            if (++b == kScratchBufs) {
                b = 0;
                sph ^= 1u;
            }
            if (!warp_wait_bar(sfull0 + 8 * b, sph, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            tc_fence_after();
            const uint32_t scr = tmem + lane_base + kScratchCol0 + (uint32_t)b * kJobRows;
            // this warp's class of the job's offset: flat entries [lo, hi)
            const int ks = job_ks(jb), first = jb.y;
            const int lo = max(first, ustart[3 * ks + sub]);
            const int hi = min(first + jb.z, ustart[3 * ks + sub + 1]);
            // 1) read this warp's scratch columns with wide loads and hand the
            //    buffer back to the MMA issuer at once;
            float v[kJobRows];
            const int ng = hi > lo ? (hi - lo + kFoldGroup - 1) / kFoldGroup : 0;  // <= 3
            if (ng > 0) tmem_ld_x16(scr + (uint32_t)(lo - first), v);
            if (ng > 1) tmem_ld_x16(scr + (uint32_t)(lo - first + kFoldGroup), v + kFoldGroup);
            if (ng > 2) tmem_ld_x16(scr + (uint32_t)(lo - first + 2 * kFoldGroup), v + 2 * kFoldGroup);
            tmem_wait_ld();  // the scratch values are in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty0 + 8 * b);
            // 2) then add them into the accumulator columns of their rows.
            const int ngn = hi > lo ? (hi - lo + kNarrowGroup - 1) / kNarrowGroup : 0;
            if (ngn > 0) tmem_wait_st();  // this warp's stores of the previous job have landed
#pragma unroll
            for (int gi = 0; gi < kJobRows / kNarrowGroup; ++gi) {
                if (gi < ngn) {
                    const int g0 = lo + gi * kNarrowGroup;
                    float a[kNarrowGroup];
                    uint32_t col[kNarrowGroup];
#pragma unroll
                    for (int i = 0; i < kNarrowGroup; ++i) {
                        const int e = g0 + i;
                        const uint32_t r = pr_s[min(e, hi - 1)];
                        col[i] = tmem + lane_base + (e < hi ? r : kDummyCol0 + (uint32_t)i);
                        tmem_ld_x1(col[i], a[i]);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < kNarrowGroup; ++i) tmem_st_x1(col[i], a[i] + v[gi * kNarrowGroup + i]);
                }
            }
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
    const int cap = kvol == kVol3 ? (int)m.tile_max_entries : 0;
    int sa = 0, sb = 0;
    L::depths(cap, &sa, &sb);
    if (sa < 2 || sb < 1) return SPCONV_ERR_UNSUPPORTED;
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
    // Features [n, cin] for the centre jobs: a box is one swizzle atom of channels
    // by BM rows.
    CUtensorMap xm;
    const cuuint64_t xdims[2] = {(cuuint64_t)cin, (cuuint64_t)m.n};
    const cuuint64_t xstrides[1] = {(cuuint64_t)cin * 2};
    const cuuint32_t xbox[2] = {(cuuint32_t)L::kAtomElems, (cuuint32_t)BM};
    const CUtensorMapSwizzle xswz = L::kAtomRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                    : L::kAtomRowBytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                             : CU_TENSOR_MAP_SWIZZLE_32B;
    r = enc(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), xdims, xstrides, xbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, xswz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *ce = cudaErrorInvalidValue;
        return SPCONV_ERR_CUDA;
    }
    const int smem = L::smem_bytes(cap, sa, sb);
    // The shared-memory opt-in is a property of the function in each device's
    // context, so it is set once per device (and per instantiation).
    int dev = 0;
    cudaError_t de = cudaGetDevice(&dev);
    if (de != cudaSuccess) {
        *ce = de;
        return SPCONV_ERR_CUDA;
    }
    {
        static std::mutex attr_mu;
        static std::vector<char> attr_done;
        std::lock_guard<std::mutex> lock(attr_mu);
        if (dev >= (int)attr_done.size()) attr_done.resize((size_t)dev + 1, 0);
        if (!attr_done[dev]) {
            const cudaError_t ae =
                cudaFuncSetAttribute(k_subm_tc<BM, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
            if (ae != cudaSuccess) {
                *ce = ae;
                return SPCONV_ERR_CUDA;
            }
            attr_done[dev] = 1;
        }
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
    p.tile_rows = m.tile_rows;
    p.sa = sa;
    p.sb = sb;
    p.cap = cap;
    dim3 grid((unsigned)num_tiles(m.n, m.tile_rows), (unsigned)((cout + BM - 1) / BM));
    k_subm_tc<BM, KC><<<grid, kThreads, smem, stream>>>(map, xm, p);
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
