// Fused gather -> tcgen05 GEMM -> single-write store over sorted windows.
//
// The pages fuse the 27 per-offset taps into one [N, 27*Cin] x [27*Cin, Cout]
// matmul over a cached device index (lato.2_mrp_mlx README, "Fleet benchmark"
// and the optimisation table after it).  This kernel computes the same sum,
//
//   D^T[Cout_blk, rows] = sum_k W_k^T[Cout_blk, Cin] . X_k^T[Cin, rows],
//
// laid out for sm_100a.  The map build has sorted the rows by neighbour pattern
// and recorded, per tile of consecutive sorted rows, the jobs: the centre job (all
// rows of the tile) and, per non-centre offset, spans of consecutive 16-row
// windows holding its hits, plus one contiguous stream of the jobs' source rows
// (map_window.cu).  A job is one run of MMAs whose output columns are the tile's
// own accumulator columns, so every product lands in place: no scatter, no fold,
// no atomics.  Holes inside a span are gathered as zero rows.
//
// Persistent CTAs (one per SM) take (tile, output-channel block) units from a
// work counter, so CTAs that drew cheap tiles take more of them.  Tensor memory
// holds two accumulators of 256 columns (lane = output channel, column = sorted
// row of the tile), so the epilogue of one tile overlaps the MMAs of the next.
//
// Warp roles (480 threads):
//   warp 0      TMEM allocator; lane 0 issues every tcgen05.mma and commit, from
//               commands the preparer posts (issuing blocks while the tensor pipe
//               is busy, so the issuer does nothing else)
//   warp 14     lane 0: MMA preparer: per (job, chunk) waits for the accumulator,
//               the weight tile and the gathered units, places the job in the B
//               ring and posts the command
//   warp 1      lane 0: claims units (tiles in the map's claim order, most
//               expensive first) and copies each unit's tile record (job list and
//               index-stream position) into a ring of four shared-memory slots,
//               two units ahead; then, as TMA producer, loads the weight
//               tiles W_k (A operand, MN-major straight from the [K^3 * Cin, Cout]
//               weights) into a ring of slots
//   warps 2-5   gather producers (B operand).  A tile's index stream arrives in
//               shared memory by one bulk copy, a tile ahead, into one of two
//               buffers.  The B ring is cut into units of 64 rows; a job takes
//               ceil(N / 64) consecutive units (never wrapping); each unit
//               belongs to a fixed group of gather warps (all four for
//               128-channel chunks, two otherwise), which fill every use of it
//               with 16-byte cp.async copies (zero fill for holes) into the swizzled
//               K-major layout the MMA reads, so each unit's uses are filled and
//               drained strictly in turn
//   warps 6-13  epilogue: two warps per TMEM lane quarter, alternate 32-column
//               chunks (warp w covers lanes 32 (w % 4) .. +31, the hardware's rule
//               for TMEM access): accumulator + bias -> bf16, staged in shared memory, then
//               16-byte stores to each output row, written exactly once; output
//               rows and bias are fetched before the accumulator is ready
// Every wait is bounded: after kWaitTimeoutNs the kernel records kFwdErrTimeout
// in the map's error word, stops issuing work, lets copies in flight land, waits
// (bounded) for its MMAs and frees its TMEM before returning.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace spconv {
namespace {

using namespace sm100;
using tc::kEpiGelu;
using tc::kEpiPlain;
using tc::kEpiRelu;
using tc::kEpiSilu;
using tc::kWaitTimeoutNs;
using tc::wait_bar;
using tc::warp_wait_bar;

constexpr int kWarpMma = 0, kWarpTma = 1, kWarpGather0 = 2, kGatherWarps = 4, kEpiWarps = 8;
constexpr int kWarpEpi0 = kWarpGather0 + kGatherWarps;
constexpr int kWarpPrep = kWarpEpi0 + kEpiWarps;        // 14
constexpr int kThreads = 32 * (kWarpPrep + 1);          // 480
// MMA command ring from the preparer to the issuer: per (job, chunk) two uint4,
// {A descriptor, B descriptor} and {TMEM column, instruction descriptor,
// B units | unit count << 8 | weight slot << 16 | flags << 24, accumulator buffer}.
constexpr int kCmdSlots = 16;
constexpr uint32_t kCmdRelA = 1, kCmdInit = 2, kCmdFirst = 4, kCmdTileEnd = 8, kCmdExit = 16;
constexpr int kEpiGroups = kEpiWarps / 4;  // epilogue warps per TMEM lane quarter
static_assert(kEpiWarps % 4 == 0 && kWinMaxRows / 32 % kEpiGroups == 0, "whole lane quarters, whole chunks");
constexpr int kAccBufs = 2;
constexpr int kIdxBufs = 2;
constexpr int kTileSlots = 4;          // tile-record ring
constexpr int kTileConsumers = 1 + kGatherWarps + kEpiWarps;  // arrivals that free a tile slot
constexpr int kRecBytes = kWinJobStride * 4;
constexpr int kSlotBytes = 16 + kRecBytes;  // [unit id][pad][record]
static_assert(kRecBytes % 16 == 0 && kSlotBytes % 16 == 0, "tile records are bulk-copied");
constexpr uint32_t kAccCols = kWinMaxRows;  // 256 columns per accumulator
constexpr uint32_t kTmemCols = 512;
static_assert(kAccBufs * kAccCols <= kTmemCols, "accumulators must fit TMEM");
constexpr int kUnitRows = 64;          // rows of one B-ring unit
constexpr int kMaxUnits = 32;          // the per-unit phase bits live in one 32-bit word
constexpr int kMaxASlots = 8;
constexpr int kMaxSmem = 232448;       // 227 KB opt-in limit per CTA on sm_100
constexpr int kMinSmem = 120 * 1024;   // keeps one CTA per SM: each CTA allocates all 512 TMEM columns

__host__ __device__ constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

template <int BM, int KC>
struct WinLayout {
    // B: gathered rows, K-major, split into swizzle atoms of up to 64 channels
    // (128 bytes); ring layout [atom][unit][64 rows][atom row bytes], so the rows
    // of consecutive units are contiguous for the MMA descriptor.
    static constexpr int kAtomElems = KC >= 64 ? 64 : KC;
    static constexpr int kAtoms = KC / kAtomElems;
    static constexpr int kARB = kAtomElems * 2;                // atom row bytes: 128, 64 or 32
    static constexpr int kUnitAtomBytes = kUnitRows * kARB;    // a multiple of the swizzle repeat
    static constexpr int kUnitBytes = kAtoms * kUnitAtomBytes;
    // Gather warps that fill one unit together (its rows split between them): 4
    // for 128-channel chunks, whose units are few and whose jobs wait on their fill
    // latency; 2 for narrower chunks, whose deeper rings gain from two units
    // filled at once (measured on B200: 1, 2 and 4 warps per unit).
    static constexpr int kFillWarps = KC >= 128 ? 4 : 2;
    static constexpr uint32_t kBLayout = kARB == 128 ? 2u : (kARB == 64 ? 4u : 6u);
    static constexpr uint32_t kBSbo = 8 * kARB;
    static constexpr int kStepsPerAtom = kAtomElems / 16;
    // A: weights, MN-major, BM / 64 boxes of [KC rows][64 channels], 128-byte swizzle.
    static constexpr int kABytes = BM * KC * 2;
    static constexpr int kAPad = round_up(kABytes, 1024);
    static constexpr int kChPerWarp = BM / 4;  // output channels of one TMEM lane quarter
    static constexpr int kStageRows = 16;      // output rows one epilogue warp stages at a time
    static constexpr int kStageBytes = kEpiWarps * kStageRows * kChPerWarp * 2;

    // A tile's index buffer: its stream plus one unit of slack (the last unit of a
    // job may read past the job's columns; those reads are masked).
    __host__ __device__ static int idx_buf_bytes(int max_cols) { return round_up((max_cols + kUnitRows) * 4, 128); }
    __host__ __device__ static int ring_bytes(int sa, int ub) { return sa * kAPad + ub * kUnitBytes; }
    __host__ __device__ static int num_bars(int sa, int ub) {
        return 2 * sa + 2 * ub + 2 * kAccBufs + 2 * kIdxBufs + 2 * kTileSlots + 2 * kCmdSlots + 1;
    }
    __host__ __device__ static int smem_bytes(int sa, int ub, int max_cols) {
        return 1024 + ring_bytes(sa, ub) + kStageBytes + kIdxBufs * idx_buf_bytes(max_cols) +
               kTileSlots * kSlotBytes + kCmdSlots * 32 + num_bars(sa, ub) * 8 + 16;
    }
};

struct WinParams {
    const int32_t* perm;        // [n] sorted row -> row (null: identity, kernel size 1)
    const uint32_t* recs;       // [tiles][kWinJobStride] tile records (null for kernel size 1)
    const int32_t* idx_stream;  // per-tile source rows of every job (null for kernel size 1)
    const int32_t* order;       // [tiles] claim order of the tiles (null: natural order)
    unsigned int* work;         // this launch's work counter: zero at launch, left at zero
    int64_t n, tiles;
    int rows;                   // rows per tile (multiple of 16, <= 256)
    int cblocks;                // output-channel blocks of BM
    const __nv_bfloat16* x;
    int cin;
    const __nv_bfloat16* bias;
    __nv_bfloat16* out;
    int cout;
    int act;                           // fused epilogue: spconv_act_t of conv + bias
    const __nv_bfloat16* residual;     // [n, cout] added after the activation, or null (may equal out)
    float* stats;                      // [2, cout] per-channel sum and sum of squares of out, or null
    unsigned int* err;
    int sa, ub;                 // weight-ring slots, B-ring units
    int idx_buf_elems;          // int32 entries of one tile index buffer
    int rows_tma;               // kernel size 1 with n >= 64: B units loaded as 64-row TMA tiles
};

// Waiting policy.  A waiting thread polls the barrier; while the phase is not
// complete it may back off with __nanosleep, doubling the pause up to its role's
// ceiling, so waiting warps leave the issue slots to the warps doing work.  The
// MMA roles and the producers poll without pausing: the issuer's data is usually
// about to land, and a producer that wakes late leaves a ring slot idle (measured
// on B200: 0, 32 and 128 ns ceilings give the same time on three workloads and 7%
// less on the 512-channel one without a pause).  The epilogue waits for a whole
// tile of MMAs and backs off up to 2 us.
constexpr uint32_t kSleepMma = 0, kSleepProducer = 0, kSleepEpilogue = 2048;

// B-ring units of the next (job, chunk): ceil(N / 64) consecutive units, starting
// over at unit 0 when they would run past the end.  Every role runs this on the
// same sequence, so all agree on the placement.
__device__ __forceinline__ int alloc_units(int& ucur, int ub, int ncols, int* m) {
    *m = (ncols + kUnitRows - 1) / kUnitRows;
    if (ucur + *m > ub) ucur = 0;
    const int u0 = ucur;
    ucur += *m;
    return u0;
}

// A tile slot: word 0 the claimed tile (-1: no more work), word 1 its output-channel
// block, words 4.. the tile's record.
__device__ __forceinline__ int slot_unit(const uint8_t* slot) { return *reinterpret_cast<const volatile int*>(slot); }
__device__ __forceinline__ int slot_cblk(const uint8_t* slot) {
    return *reinterpret_cast<const volatile int*>(slot + 4);
}
__device__ __forceinline__ const uint32_t* slot_rec(const uint8_t* slot) {
    return reinterpret_cast<const uint32_t*>(slot + 16);
}

template <int BM, int KC, int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    k_subm_win(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, const WinParams p) {
    using L = WinLayout<BM, KC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int SA = p.sa, UB = p.ub;
    uint8_t* a_ring = smem;
    uint8_t* b_ring = smem + SA * L::kAPad;
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(b_ring + UB * L::kUnitBytes);
    int32_t* idx_buf = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(stage) + L::kStageBytes);
    uint8_t* tile_ring = reinterpret_cast<uint8_t*>(idx_buf + kIdxBufs * p.idx_buf_elems);
    uint4* cmd_ring = reinterpret_cast<uint4*>(tile_ring + kTileSlots * kSlotBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(cmd_ring + 2 * kCmdSlots);
    int* misc = reinterpret_cast<int*>(bars + L::num_bars(SA, UB));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_flag = misc + 1;

    const uint32_t fullA0 = smem_addr(bars), emptyA0 = fullA0 + 8 * SA;
    const uint32_t fullB0 = emptyA0 + 8 * SA, emptyB0 = fullB0 + 8 * UB;
    const uint32_t accF0 = emptyB0 + 8 * UB, accE0 = accF0 + 8 * kAccBufs;
    const uint32_t idxF0 = accE0 + 8 * kAccBufs, idxE0 = idxF0 + 8 * kIdxBufs;
    const uint32_t tileF0 = idxE0 + 8 * kIdxBufs, tileE0 = tileF0 + 8 * kTileSlots;
    const uint32_t cmdF0 = tileE0 + 8 * kTileSlots, cmdE0 = cmdF0 + 8 * kCmdSlots;
    const uint32_t drain = cmdE0 + 8 * kCmdSlots;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = p.cin / KC;
    const int64_t units = p.tiles * p.cblocks;

    if (threadIdx.x == kWarpTma * 32) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(fullA0 + 8 * s, 1);
            mbar_init(emptyA0 + 8 * s, 1);
        }
        for (int u = 0; u < UB; ++u) {
            // cp.async fill: every lane of the unit's filling warps; TMA tile: the
            // issuing thread's expect-tx arrival, then the bytes
            mbar_init(fullB0 + 8 * u, p.rows_tma ? 1 : 32 * L::kFillWarps);
            mbar_init(emptyB0 + 8 * u, 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(accF0 + 8 * b, 1);
            mbar_init(accE0 + 8 * b, kEpiWarps);
        }
        for (int b = 0; b < kIdxBufs; ++b) {
            mbar_init(idxF0 + 8 * b, 1);
            mbar_init(idxE0 + 8 * b, kGatherWarps);
        }
        for (int s = 0; s < kTileSlots; ++s) {
            mbar_init(tileF0 + 8 * s, 1);
            mbar_init(tileE0 + 8 * s, kTileConsumers);
        }
        for (int s = 0; s < kCmdSlots; ++s) {
            mbar_init(cmdF0 + 8 * s, 1);
            mbar_init(cmdE0 + 8 * s, 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool aborted = false;

    if (warp == kWarpMma) {
        // ------------------------------------------------ tcgen05.mma issuer (lane 0)
        // Issuing blocks while the tensor pipe is busy, so this thread does nothing
        // else: it takes each (job, chunk) command the preparer posted, issues the
        // MMAs and the commits that release the operands, and moves on.
        if (lane == 0) {
            for (int cq = 0;; ++cq) {
                const int s = cq % kCmdSlots;
                if (!wait_bar<kSleepMma>(cmdF0 + 8 * s, (uint32_t)(cq / kCmdSlots) & 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                const uint4 c0 = cmd_ring[2 * s], c1 = cmd_ring[2 * s + 1];
                mbar_arrive(cmdE0 + 8 * s);  // the command is in registers now
                const uint32_t fl = c1.z >> 24;
                if (fl & kCmdExit) break;
                if (fl & kCmdFirst) tc_fence_after();  // the epilogue's reads of this accumulator are done
                // the B units were written by cp.async (generic proxy); the MMA reads
                // them through the async proxy
                fence_proxy_async_smem();
                const uint64_t adesc0 = (uint64_t)c0.x | ((uint64_t)c0.y << 32);
                const uint64_t bdesc0 = (uint64_t)c0.z | ((uint64_t)c0.w << 32);
                // later K steps add their byte offset (>> 4) to the start-address field,
                // which cannot carry out of it because shared addresses stay below 256 KB
#pragma unroll
                for (int kk = 0; kk < KC / 16; ++kk) {
                    const uint32_t boff =
                        (uint32_t)((kk / L::kStepsPerAtom) * UB * L::kUnitAtomBytes + (kk % L::kStepsPerAtom) * 32);
                    mma_bf16(c1.x, adesc0 + (uint64_t)((kk * 2048) >> 4), bdesc0 + (uint64_t)(boff >> 4), c1.y,
                             ((fl & kCmdInit) && kk == 0) ? 0u : 1u);
                }
                const int u0 = (int)(c1.z & 0xFFu), m = (int)((c1.z >> 8) & 0xFFu), as = (int)((c1.z >> 16) & 0xFFu);
                for (int q = 0; q < m; ++q) mma_commit(emptyB0 + 8 * (u0 + q));
                if (fl & kCmdRelA) mma_commit(emptyA0 + 8 * as);
                if (fl & kCmdTileEnd) mma_commit(accF0 + 8 * c1.w);
            }
            if (aborted) {
                mma_commit(drain);  // wait for the MMAs in flight before TMEM is freed
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == kWarpPrep) {
        // ------------------------------------------------ MMA preparer (lane 0)
        // Walks the tiles and their jobs: waits for the accumulator, the weight tile
        // and the gathered units of each (job, chunk), places it in the B ring and
        // posts one command per (job, chunk) to the issuer, up to kCmdSlots ahead.
        if (lane == 0) {
            int as = SA - 1;
            uint32_t aph = 1u;
            int ucur = 0;
            uint32_t bph = 0;  // bit u: phase of unit u's next use
            int cq = 0;
            auto post = [&](const uint4& c0, const uint4& c1) -> bool {
                const int s = cq % kCmdSlots;
                if (!wait_bar<kSleepMma>(cmdE0 + 8 * s, ((uint32_t)(cq / kCmdSlots) & 1u) ^ 1u, abort_flag, p.err))
                    return false;
                cmd_ring[2 * s] = c0;
                cmd_ring[2 * s + 1] = c1;
                mbar_arrive(cmdF0 + 8 * s);
                ++cq;
                return true;
            };
            for (int i = 0; !aborted; ++i) {
                const int s = i % kTileSlots;
                const uint8_t* slot = tile_ring + s * kSlotBytes;
                if (!wait_bar<kSleepMma>(tileF0 + 8 * s, (uint32_t)(i / kTileSlots) & 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                if (slot_unit(slot) < 0) {
                    if (!post(make_uint4(0, 0, 0, 0), make_uint4(0, 0, kCmdExit << 24, 0))) aborted = true;
                    break;
                }
                const uint32_t* rec = slot_rec(slot);
                const int buf = i & 1;
                if (!wait_bar<kSleepMma>(accE0 + 8 * buf, ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                const uint32_t dbase = tmem + (uint32_t)buf * kAccCols;
                const int nj = (int)rec[0];
                int prev_k = -1;
                uint32_t jw = rec[kWinRecHeader];
                for (int j = 0; j < nj && !aborted; ++j) {
                    const uint32_t jn = j + 1 < nj ? rec[kWinRecHeader + j + 1] : 0xFFFFFFFFu;
                    const int k = win_job_k(jw), w0 = win_job_w0(jw), ncols = win_job_nw(jw) * kWinCols;
                    const bool new_k = k != prev_k;
                    prev_k = k;
                    const bool last_of_k = jn == 0xFFFFFFFFu || win_job_k(jn) != k;
                    const uint32_t idesc = idesc_bf16(BM, (uint32_t)ncols);
                    const uint32_t d = dbase + (uint32_t)(w0 * kWinCols);
                    for (int c = 0; c < nchunks; ++c) {
                        if (nchunks > 1 || (c == 0 && new_k)) {
                            if (++as == SA) {
                                as = 0;
                                aph ^= 1u;
                            }
                            if (!wait_bar<kSleepMma>(fullA0 + 8 * as, aph, abort_flag, p.err)) {
                                aborted = true;
                                break;
                            }
                        }
                        int m = 0;
                        const int u0 = alloc_units(ucur, UB, ncols, &m);
                        for (int q = 0; q < m; ++q) {
                            if (!wait_bar<kSleepMma>(fullB0 + 8 * (u0 + q), (bph >> (u0 + q)) & 1u, abort_flag,
                                                     p.err)) {
                                aborted = true;
                                break;
                            }
                        }
                        if (aborted) break;
                        const uint64_t adesc0 = smem_desc(smem_addr(a_ring + as * L::kAPad), KC * 128, 1024, 2);
                        const uint64_t bdesc0 = smem_desc(smem_addr(b_ring) + (uint32_t)(u0 * L::kUnitAtomBytes), 16,
                                                          L::kBSbo, L::kBLayout);
                        uint32_t fl = 0;
                        if (nchunks > 1 || last_of_k) fl |= kCmdRelA;
                        if (j == 0 && c == 0) fl |= kCmdInit | kCmdFirst;
                        if (j == nj - 1 && c == nchunks - 1) fl |= kCmdTileEnd;
                        const uint4 c0 = make_uint4((uint32_t)adesc0, (uint32_t)(adesc0 >> 32), (uint32_t)bdesc0,
                                                    (uint32_t)(bdesc0 >> 32));
                        const uint4 c1 = make_uint4(d, idesc, (uint32_t)u0 | ((uint32_t)m << 8) |
                                                                   ((uint32_t)as << 16) | (fl << 24),
                                                    (uint32_t)buf);
                        if (!post(c0, c1)) {
                            aborted = true;
                            break;
                        }
                        for (int q = 0; q < m; ++q) bph ^= 1u << (u0 + q);
                    }
                    jw = jn;
                }
                if (aborted) break;
                mbar_arrive(tileE0 + 8 * s);
            }
        }
        __syncwarp();
    } else if (warp == kWarpTma) {
        // ------------------------------------------------ scheduler + weight tiles (lane 0)
        if (lane == 0) {
            // Claim unit number idx into slot idx % kTileSlots once all consumers have
            // released that slot's previous unit; no unit left: a -1 marker.
            auto push = [&](int idx) -> bool {
                const int s = idx % kTileSlots;
                uint8_t* slot = tile_ring + s * kSlotBytes;
                if (!wait_bar<kSleepProducer>(tileE0 + 8 * s, ((uint32_t)(idx / kTileSlots) & 1u) ^ 1u, abort_flag,
                                              p.err))
                    return false;
                const unsigned int c = atomicAdd(p.work, 1u);  // claim number: tile order, then channel block
                int* su = reinterpret_cast<int*>(slot);
                if ((int64_t)c >= units) {
                    // every CTA claims until its first miss, so a launch makes exactly
                    // units + gridDim.x claims; the CTA that makes the last one knows
                    // that no claim is pending and sets the counter back to zero for
                    // the next launch that uses it
                    if ((int64_t)c == units + gridDim.x - 1) atomicExch(p.work, 0u);
                    su[0] = -1;
                    mbar_arrive(tileF0 + 8 * s);
                    return false;
                }
                const int64_t t = p.order ? (int64_t)p.order[c / p.cblocks] : (int64_t)(c / p.cblocks);
                su[0] = (int)t;
                su[1] = (int)(c % p.cblocks);
                if (p.recs) {
                    mbar_arrive_expect_tx(tileF0 + 8 * s, kRecBytes);
                    bulk_load(smem_addr(slot + 16), p.recs + t * kWinJobStride, kRecBytes, tileF0 + 8 * s);
                } else {  // kernel size 1: one centre job over the tile, no index stream
                    uint32_t* r = reinterpret_cast<uint32_t*>(slot + 16);
                    r[0] = 1u;
                    r[1] = 0u;
                    r[kWinRecHeader] = win_job(0, 0, p.rows / kWinCols);
                    mbar_arrive(tileF0 + 8 * s);
                }
                return true;
            };
            // claims run two units ahead of the weight loads
            bool more = push(0) && push(1);
            int s_a = 0;  // weight slot and phase
            uint32_t ph = 0;
            for (int i = 0; !aborted; ++i) {
                if (more) more = push(i + 2);
                if (*abort_flag) {
                    aborted = true;
                    break;
                }
                const int s = i % kTileSlots;
                const uint8_t* slot = tile_ring + s * kSlotBytes;
                if (!wait_bar<kSleepProducer>(tileF0 + 8 * s, (uint32_t)(i / kTileSlots) & 1u, abort_flag, p.err)) {
                    aborted = true;
                    break;
                }
                if (slot_unit(slot) < 0) break;
                const int cblk = slot_cblk(slot);
                const uint32_t* rec = slot_rec(slot);
                const int nj = (int)rec[0];
                int prev_k = -1;
                for (int j = 0; j < nj && !aborted; ++j) {
                    const int k = win_job_k(rec[kWinRecHeader + j]);
                    const bool new_k = k != prev_k;
                    prev_k = k;
                    if (nchunks == 1 && !new_k) continue;  // the loaded tile serves this job too
                    for (int c = 0; c < nchunks; ++c) {
                        if (!wait_bar<kSleepProducer>(emptyA0 + 8 * s_a, ph ^ 1u, abort_flag, p.err)) {
                            aborted = true;
                            break;
                        }
                        const uint32_t dst = smem_addr(a_ring + s_a * L::kAPad);
                        mbar_arrive_expect_tx(fullA0 + 8 * s_a, L::kABytes);
                        const int y = k * p.cin + c * KC;
                        for (int box = 0; box < BM / 64; ++box)
                            tma_load_2d(dst + box * KC * 128, &wmap, cblk * BM + box * 64, y, fullA0 + 8 * s_a);
                        if (++s_a == SA) {
                            s_a = 0;
                            ph ^= 1u;
                        }
                    }
                }
            }
            if (aborted) __nanosleep(200000);  // let loads in flight land before the CTA exits
        }
        __syncwarp();
    } else if (warp < kWarpEpi0) {
        // ------------------------------------------------ gather producers
        // The gather warps form kGroups groups of kFillWarps; unit u belongs to
        // group u % kGroups, whose warps fill every use of it (warp sub of the group
        // its slice of kSliceRows rows), so kGroups units fill at once.  Every use
        // of a unit is thus waited for and filled by the same warps, in order: no
        // warp reaches a unit's next use before the previous one was released,
        // which the phase-parity wait could not tell apart from the use before it.
        // Lane l copies 16-byte chunk l % kThreadsPerRow of rows
        // l / kThreadsPerRow + kWarpRows * pass of its slice.
        constexpr int kThreadsPerRow = KC * 2 / 16;                // 16-byte chunks of one row's chunk
        constexpr int kWarpRows = 32 / kThreadsPerRow;             // rows one warp instruction covers
        constexpr int kSliceRows = kUnitRows / L::kFillWarps;      // rows of a unit one warp fills
        constexpr int kGroups = kGatherWarps / L::kFillWarps;      // groups of warps that share units
        // passes of one warp instruction over its slice, taken kBatch at a time; when
        // one instruction covers more rows than a slice holds, lanes past it idle
        constexpr int kPasses = kSliceRows >= kWarpRows ? kSliceRows / kWarpRows : 1;
        constexpr int kBatch = kPasses < 8 ? kPasses : 8;
        static_assert(kSliceRows % kWarpRows == 0 || kWarpRows % kSliceRows == 0, "slices and passes must align");
        static_assert(kPasses % kBatch == 0, "batches must tile the passes");
        constexpr int kChunksPerAtom = L::kARB / 16;
        constexpr uint32_t kSwz = L::kARB / 16 - 1;
        const int g = warp - kWarpGather0;
        const int grp = g / L::kFillWarps, sub = g % L::kFillWarps;  // unit group, slice within a unit
        const int q = lane % kThreadsPerRow;
        const int prow = lane / kThreadsPerRow;
        const int atom = q / kChunksPerAtom, qa = q % kChunksPerAtom;
        const bool issuer = g == 0 && p.idx_stream != nullptr;  // fetches the index streams
        int ucur = 0;
        uint32_t bph = 0;
        // the index stream of tile number i goes to buffer i & 1, free once every
        // gather warp has finished tile number i - 2
        auto fetch_idx = [&](int i) -> bool {
            const int s = i % kTileSlots;
            const uint8_t* slot = tile_ring + s * kSlotBytes;
            if (!warp_wait_bar<kSleepProducer>(tileF0 + 8 * s, (uint32_t)(i / kTileSlots) & 1u, abort_flag, p.err))
                return false;
            if (slot_unit(slot) < 0) return true;  // no such tile
            const int b = i & 1;
            if (!warp_wait_bar<kSleepProducer>(idxE0 + 8 * b, ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, p.err))
                return false;
            if (lane == 0) {
                const uint32_t* rec = slot_rec(slot);
                const uint32_t bytes = rec[1] * 4u;
                const int64_t s0 = (int64_t)((uint64_t)rec[2] | ((uint64_t)rec[3] << 32));
                mbar_arrive_expect_tx(idxF0 + 8 * b, bytes);
                bulk_load(smem_addr(idx_buf + b * p.idx_buf_elems), p.idx_stream + s0, bytes, idxF0 + 8 * b);
            }
            __syncwarp();
            return true;
        };
        if (issuer && !fetch_idx(0)) aborted = true;
        for (int i = 0; !aborted; ++i) {
            const int s = i % kTileSlots;
            const uint8_t* slot = tile_ring + s * kSlotBytes;
            if (!warp_wait_bar<kSleepProducer>(tileF0 + 8 * s, (uint32_t)(i / kTileSlots) & 1u, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            const int u = slot_unit(slot);
            if (u < 0) break;
            if (issuer && !fetch_idx(i + 1)) {
                aborted = true;
                break;
            }
            const int buf = i & 1;
            if (p.idx_stream &&
                !warp_wait_bar<kSleepProducer>(idxF0 + 8 * buf, (uint32_t)(i >> 1) & 1u, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            const int32_t* ibuf = idx_buf + buf * p.idx_buf_elems;
            const int64_t row_t0 = (int64_t)u * p.rows;
            const uint32_t* rec = slot_rec(slot);
            const int nj = (int)rec[0];
            int joff = 0;  // the job's first entry in the tile's index stream
            for (int j = 0; j < nj && !aborted; ++j) {
                const uint32_t jw = rec[kWinRecHeader + j];
                const int ncols = win_job_nw(jw) * kWinCols;
                const int64_t r0 = row_t0 + win_job_w0(jw) * kWinCols;  // first sorted row of the job
                for (int c = 0; c < nchunks && !aborted; ++c) {
                    int m = 0;
                    const int u0 = alloc_units(ucur, UB, ncols, &m);
                    const __nv_bfloat16* xc = p.x + c * KC + q * 8;
                    for (int qq = 0; qq < m; ++qq) {
                        const int unit = u0 + qq;
                        if (unit % kGroups != grp) continue;  // another group's unit
                        if (p.rows_tma) {
                            // kernel size 1: the job's rows are consecutive input rows, so
                            // the unit is one 64-row tile per channel atom (rows past n
                            // read as zeros); the group's first warp loads it
                            if (sub != 0) continue;
                            if (!warp_wait_bar<kSleepProducer>(emptyB0 + 8 * unit, ((bph >> unit) & 1u) ^ 1u,
                                                               abort_flag, p.err)) {
                                aborted = true;
                                break;
                            }
                            if (lane == 0) {
                                const uint32_t full = fullB0 + 8 * unit;
                                mbar_arrive_expect_tx(full, (uint32_t)L::kUnitBytes);
#pragma unroll
                                for (int at = 0; at < L::kAtoms; ++at)
                                    tma_load_2d(smem_addr(b_ring) + (uint32_t)((at * UB + unit) * L::kUnitAtomBytes),
                                                &xmap, c * KC + at * L::kAtomElems, (int)(r0 + qq * kUnitRows), full);
                            }
                            __syncwarp();
                            continue;
                        }
                        if (!warp_wait_bar<kSleepProducer>(emptyB0 + 8 * unit, ((bph >> unit) & 1u) ^ 1u, abort_flag,
                                                           p.err)) {
                            aborted = true;
                            break;
                        }
                        const uint32_t ubase = smem_addr(b_ring) + (uint32_t)(atom * UB * L::kUnitAtomBytes) +
                                               (uint32_t)(unit * L::kUnitAtomBytes);
                        // kBatch passes at a time: their source rows first (rows past the
                        // job read as holes, so no pass branches), then their copies
#pragma unroll 1
                        for (int p0 = 0; p0 < kPasses; p0 += kBatch) {
                            int src[kBatch];
#pragma unroll
                            for (int pp = 0; pp < kBatch; ++pp) {
                                const int r = qq * kUnitRows + sub * kSliceRows + prow + (p0 + pp) * kWarpRows;
                                if (p.idx_stream) {
                                    const int v = ibuf[joff + r];
                                    src[pp] = r < ncols ? v : -1;
                                } else {
                                    const int64_t rr = r0 + r;
                                    src[pp] = r < ncols && rr < p.n ? (int)rr : -1;
                                }
                            }
#pragma unroll
                            for (int pp = 0; pp < kBatch; ++pp) {
                                if (kWarpRows > kSliceRows && prow >= kSliceRows) continue;
                                const uint32_t lin =
                                    (uint32_t)((sub * kSliceRows + prow + (p0 + pp) * kWarpRows) * L::kARB + qa * 16);
                                cp_async_16(ubase + (lin ^ (((lin >> 7) & kSwz) << 4)),
                                            xc + (int64_t)(src[pp] >= 0 ? src[pp] : 0) * p.cin, src[pp] >= 0 ? 16u : 0u);
                            }
                        }
                        cp_async_mbar_arrive_noinc(fullB0 + 8 * unit);
                    }
                    for (int qq = 0; qq < m; ++qq) bph ^= 1u << (u0 + qq);
                }
                joff += ncols;
            }
            __syncwarp();
            if (lane == 0) {
                if (p.idx_stream) mbar_arrive(idxE0 + 8 * buf);  // this warp is done with the tile's indices
                mbar_arrive(tileE0 + 8 * s);
            }
        }
        // copies in flight (an index stream, row tiles) land before the CTA exits
        if ((issuer || p.rows_tma) && aborted && lane == 0) __nanosleep(200000);
        cp_async_wait_all();
    } else if (warp < kWarpEpi0 + kEpiWarps) {
        // ------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int half = (warp - kWarpEpi0) >> 2;  // this warp's group within its lane quarter
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        __nv_bfloat16* stg = stage + (warp - kWarpEpi0) * L::kStageRows * L::kChPerWarp;
        constexpr int kChunksPerWarp = kWinMaxRows / 32 / kEpiGroups;  // this warp's 32-column chunks of a tile
        const bool lane_ok = lane < L::kChPerWarp;
        const tc::EpiOut eo{p.out, p.residual, p.cout, p.act};
        for (int i = 0; !aborted; ++i) {
            const int s = i % kTileSlots;
            const uint8_t* slot = tile_ring + s * kSlotBytes;
            if (!warp_wait_bar<kSleepEpilogue>(tileF0 + 8 * s, (uint32_t)(i / kTileSlots) & 1u, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            const int u = slot_unit(slot);
            __syncwarp();
            if (lane == 0) mbar_arrive(tileE0 + 8 * s);  // only the unit number is needed here
            if (u < 0) break;
            const int64_t t = u;
            const int cblk = slot_cblk(slot);
            const int buf = i & 1;
            const int ch_base = cblk * BM + quarter * L::kChPerWarp;
            const int64_t row_t0 = t * p.rows;
            const int t_eff = (int)min((int64_t)p.rows, p.n - row_t0);
            // output rows and bias first: their loads overlap the wait for the MMAs
            // (columns at or past t_eff are not this tile's rows)
            int orow[kChunksPerWarp];
#pragma unroll
            for (int c4 = 0; c4 < kChunksPerWarp; ++c4) {
                const int col = (half + kEpiGroups * c4) * 32 + lane;
                orow[c4] = col < t_eff ? (p.perm ? p.perm[row_t0 + col] : (int)(row_t0 + col)) : -1;
            }
            const float bv = (p.bias && lane_ok) ? __bfloat162float(p.bias[ch_base + lane]) : 0.0f;
            if constexpr (kEpi != kEpiPlain) {
                // the residual slices of this warp's rows into L2 while the MMAs run
                if (p.residual) {
#pragma unroll
                    for (int c4 = 0; c4 < kChunksPerWarp; ++c4)
                        if (orow[c4] >= 0) prefetch_l2(p.residual + (int64_t)orow[c4] * p.cout + ch_base);
                }
            }
            if (!warp_wait_bar<kSleepEpilogue>(accF0 + 8 * buf, (uint32_t)(i >> 1) & 1u, abort_flag, p.err)) {
                aborted = true;
                break;
            }
            tc_fence_after();
            float s1 = 0.0f, s2 = 0.0f;  // this lane's channel statistics over the tile (fused epilogue)
#pragma unroll
            for (int c4 = 0; c4 < kChunksPerWarp; ++c4) {
                const int cc = half + kEpiGroups * c4;
                if (cc * 32 < t_eff) {
                    float v[32];
                    tmem_ld_x32(tmem + lane_base + (uint32_t)buf * kAccCols + (uint32_t)(cc * 32), v);
                    tmem_wait_ld();
                    tc::store_chunk<kEpi, L::kChPerWarp, L::kStageRows>(v, orow[c4], lane, lane_ok, bv, ch_base,
                                                                        cc * 32, t_eff, eo, stg, s1, s2);
                }
            }
            if constexpr (kEpi != kEpiPlain) {
                if (p.stats && lane_ok) {
                    atomicAdd(p.stats + ch_base + lane, s1);
                    atomicAdd(p.stats + p.cout + ch_base + lane, s2);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accE0 + 8 * buf);
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

int g_force_sa = 0, g_force_ub = 0;  // test hook: ring depths (0 = automatic)

// Ring depths: three weight slots (two if that leaves too few units), then as
// many B units as fit (at most kMaxUnits), then any room left to weight slots (at
// most kMaxASlots); a tile's centre job needs ceil(rows / 64) units at once.
// max_cols sizes the two tile index buffers.
template <int BM, int KC>
bool choose_depths(int rows, int max_cols, int* sa, int* ub) {
    using L = WinLayout<BM, KC>;
    const int need = (rows + kUnitRows - 1) / kUnitRows;
    if (g_force_sa > 0 && g_force_ub > 0) {
        *sa = g_force_sa;
        *ub = g_force_ub;
        return *ub >= need && *ub <= kMaxUnits && *sa <= kMaxASlots && L::smem_bytes(*sa, *ub, max_cols) <= kMaxSmem;
    }
    for (int a = 3; a >= 2; --a) {
        int b = 0;
        while (b < kMaxUnits && L::smem_bytes(a, b + 1, max_cols) <= kMaxSmem) ++b;
        if (b >= need + 1 || (a == 2 && b >= need)) {
            while (a < kMaxASlots && L::smem_bytes(a + 1, b, max_cols) <= kMaxSmem) ++a;
            *sa = a;
            *ub = b;
            return true;
        }
    }
    return false;
}

template <int BM, int KC>
spconv_status_t launch(const MapData& m, const void* x, int cin, const void* w, const void* bias, void* out,
                       int cout, const Epilogue& epi, cudaStream_t stream, cudaError_t* ce) {
    using L = WinLayout<BM, KC>;
    tc::EncodeTiledFn enc = tc::encode_fn();
    if (!enc) {
        *ce = cudaErrorSymbolNotFound;
        return SPCONV_ERR_CUDA;
    }
    const int kvol = m.kernel_size == 3 ? kVol3 : 1;
    const int max_cols = kvol == kVol3 ? (int)m.max_tile_cols : 0;
    int sa = 0, ub = 0;
    if (!choose_depths<BM, KC>(m.win_rows, max_cols, &sa, &ub)) return SPCONV_ERR_UNSUPPORTED;
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
    // Features [n, cin] as 64-row tiles of one channel atom, for kernel size 1 (no
    // gather: a job's rows are consecutive); swizzled like the B ring.  Encoded
    // only when used, and then n >= 64 (one tile at most as tall as the tensor).
    CUtensorMap xmap;
    memset(&xmap, 0, sizeof(xmap));
    const bool rows_tma = kvol == 1 && m.n >= kUnitRows;
    if (rows_tma) {
        const cuuint64_t xdims[2] = {(cuuint64_t)cin, (cuuint64_t)m.n};
        const cuuint64_t xstrides[1] = {(cuuint64_t)cin * 2};
        const cuuint32_t xbox[2] = {(cuuint32_t)L::kAtomElems, (cuuint32_t)kUnitRows};
        const CUtensorMapSwizzle xswz = L::kARB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                        : (L::kARB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                                         : CU_TENSOR_MAP_SWIZZLE_32B);
        r = enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), xdims, xstrides, xbox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, xswz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            *ce = cudaErrorInvalidValue;
            return SPCONV_ERR_CUDA;
        }
    }
    const int need_smem = L::smem_bytes(sa, ub, max_cols);
    const int smem = need_smem > kMinSmem ? need_smem : kMinSmem;
    int dev = 0;
    cudaError_t de = cudaGetDevice(&dev);
    if (de != cudaSuccess) {
        *ce = de;
        return SPCONV_ERR_CUDA;
    }
    // the fused-epilogue instantiation runs only when an epilogue op is asked for,
    // so plain layers keep the plain store
    const int kind = tc::epi_kind(epi);
    auto kernel = kind == kEpiPlain  ? k_subm_win<BM, KC, kEpiPlain>
                  : kind == kEpiRelu ? k_subm_win<BM, KC, kEpiRelu>
                  : kind == kEpiSilu ? k_subm_win<BM, KC, kEpiSilu>
                                     : k_subm_win<BM, KC, kEpiGelu>;
    {   // the shared-memory opt-in is per device context and instantiation
        static std::mutex attr_mu;
        static std::vector<char> attr_done;  // bit k: epilogue instantiation k
        std::lock_guard<std::mutex> lock(attr_mu);
        if (dev >= (int)attr_done.size()) attr_done.resize((size_t)dev + 1, 0);
        const char bit = (char)(1 << kind);
        if (!(attr_done[dev] & bit)) {
            const cudaError_t ae = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
            if (ae != cudaSuccess) {
                *ce = ae;
                return SPCONV_ERR_CUDA;
            }
            attr_done[dev] |= bit;
        }
    }
    // this launch's work counter: one of the map's slots in turn (zeroed by the
    // build, and set back to zero by the launch's last claim)
    static std::atomic<uint64_t> launches{0};
    unsigned int* work = m.sched + (launches.fetch_add(1) % kSchedSlots);
    WinParams p;
    p.perm = kvol == kVol3 ? m.perm : nullptr;
    p.recs = kvol == kVol3 ? m.win_jobs : nullptr;
    p.idx_stream = kvol == kVol3 ? m.idx_stream : nullptr;
    p.order = kvol == kVol3 ? m.win_order : nullptr;
    p.work = work;
    p.n = m.n;
    p.tiles = m.win_tiles;
    p.rows = m.win_rows;
    p.cblocks = cout / BM;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.cin = cin;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.cout = cout;
    p.err = m.fwd_err;
    p.sa = sa;
    p.ub = ub;
    p.idx_buf_elems = L::idx_buf_bytes(max_cols) / 4;
    p.rows_tma = rows_tma ? 1 : 0;
    p.act = epi.act;
    p.residual = static_cast<const __nv_bfloat16*>(epi.residual);
    p.stats = epi.stats;
    const int64_t units = m.win_tiles * p.cblocks;
    const int64_t grid = units < m.num_sms ? units : m.num_sms;
    kernel<<<(unsigned)grid, kThreads, smem, stream>>>(map, xmap, p);
    *ce = cudaGetLastError();
    return *ce == cudaSuccess ? SPCONV_OK : SPCONV_ERR_CUDA;
}

}  // namespace

void set_forced_ring_depths(int sa, int ub) {
    g_force_sa = sa;
    g_force_ub = ub;
}

spconv_status_t launch_forward_tcgen05(const MapData& m, const void* x, int cin, const void* w, const void* bias,
                                       void* out, int cout, const Epilogue& epi, cudaStream_t stream,
                                       cudaError_t* ce) {
    *ce = cudaSuccess;
    if (cin % 16 != 0 || cout % 64 != 0) return SPCONV_ERR_UNSUPPORTED;
    if (m.n == 0) return SPCONV_OK;
    const bool bm128 = cout % 128 == 0;
    const int kc = cin % 128 == 0 ? 128 : (cin % 64 == 0 ? 64 : (cin % 32 == 0 ? 32 : 16));
    if (bm128) {
        if (kc == 128) return launch<128, 128>(m, x, cin, w, bias, out, cout, epi, stream, ce);
        if (kc == 64) return launch<128, 64>(m, x, cin, w, bias, out, cout, epi, stream, ce);
        if (kc == 32) return launch<128, 32>(m, x, cin, w, bias, out, cout, epi, stream, ce);
        return launch<128, 16>(m, x, cin, w, bias, out, cout, epi, stream, ce);
    }
    if (kc == 128) return launch<64, 128>(m, x, cin, w, bias, out, cout, epi, stream, ce);
    if (kc == 64) return launch<64, 64>(m, x, cin, w, bias, out, cout, epi, stream, ce);
    if (kc == 32) return launch<64, 32>(m, x, cin, w, bias, out, cout, epi, stream, ce);
    return launch<64, 16>(m, x, cin, w, bias, out, cout, epi, stream, ce);
}

}  // namespace spconv
