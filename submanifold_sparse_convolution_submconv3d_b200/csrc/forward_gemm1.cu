// Kernel size 1: a weight-stationary tcgen05 GEMM over the active rows.
//
// With a single offset the submanifold convolution is a plain product,
// out = x . W[0] + bias, row by row (the lato.2_mrp_mlx README, "Status", lists
// SubMConv3d with kernel size 1 beside kernel size 3).  The rows need no map and
// no gather; this kernel computes
//
//   D^T[Cout_blk, rows] = W^T[Cout_blk, Cin] . X^T[Cin, rows]
//
// with D transposed in tensor memory (lane = output channel, column = row) like
// the window kernel, so the two share the epilogue.
//
// Each CTA owns one block of BM output channels for the whole launch.  Its slice
// of the weights (Cin x BM bf16) is loaded into shared memory once, one barrier
// per 64-channel chunk so the first MMAs start on the first chunk; the CTA then
// streams 128-row tiles of x through a ring of [128 rows x 64 channels] stages.
//
// The CTAs of one row slot (one per output-channel block, launched next to each
// other) read the same x tile at about the same time, so x comes from HBM about
// once; what bounds the kernel is the rate at which the x stages reach the SMs
// from L2, not the tensor pipe.
//
// Warp roles (320 threads):
//   warp 0     TMEM allocator; lane 0 issues the MMAs (M = BM, N = 128, K = 16)
//              and the commits that free x stages and hand accumulators over
//   warp 1     lane 0: TMA producer: the weight slice, then the x stages
//   warps 2-9  epilogue: two warps per TMEM lane quarter, one 32-column chunk
//              each of the two in its half of a tile; four accumulators of 128
//              columns let the epilogue trail the MMAs by up to three tiles
// Every wait is bounded as in the window kernel: after the time limit the kernel
// records kFwdErrTimeout, stops, lets its copies land, waits (bounded) for its
// MMAs and frees its TMEM.
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

constexpr int kRows = 128;          // rows per tile: the MMA's N
constexpr int kChunk = 64;          // input channels per stage: one 128-byte swizzle atom
constexpr int kAccBufs = 4;         // accumulators of kRows TMEM columns
constexpr uint32_t kTmemCols = kAccBufs * kRows;
static_assert(kTmemCols == 512, "four accumulators fill the tensor memory");
constexpr int kWarpMma = 0, kWarpTma = 1, kWarpEpi0 = 2, kEpiWarps = 8;
constexpr int kThreads = 32 * (kWarpEpi0 + kEpiWarps);  // 320
constexpr int kChunksPerWarp = kRows / 32 / 2;          // two warps per lane quarter
constexpr int kXStageBytes = kRows * kChunk * 2;        // 16 KB
constexpr int kMinStages = 2, kMaxStages = 8;
constexpr int kMaxWChunks = 23;  // 1472 input channels: the largest slice that fits (64 output channels)
constexpr int kMaxSmem = 232448;
constexpr uint32_t kSleepEpilogue = 2048;

template <int BM>
struct G1Layout {
    static constexpr int kWChunkBytes = BM * kChunk * 2;  // BM / 64 boxes of [64 input][64 output channels]
    static constexpr int kChPerWarp = BM / 4;             // output channels of one TMEM lane quarter
    static constexpr int kStageRows = 16;
    static constexpr int kStgBytes = kEpiWarps * kStageRows * kChPerWarp * 2;
    // weight chunks; per stage full and empty; per accumulator full and empty; drain
    __host__ __device__ static int num_bars(int wch, int stages) { return wch + 2 * stages + 2 * kAccBufs + 1; }
    __host__ __device__ static int smem_bytes(int cin, int stages) {
        const int wch = cin / kChunk;
        return 1024 + wch * kWChunkBytes + stages * kXStageBytes + kStgBytes + num_bars(wch, stages) * 8 + 16;
    }
};

struct G1Params {
    int64_t n;
    int cin, cout, cblocks, stages;
    const __nv_bfloat16* bias;
    __nv_bfloat16* out;
    int act;
    const __nv_bfloat16* residual;
    float* stats;
    unsigned int* err;
};

// Bounded poll used only after an abort, to let copies in flight land.
__device__ __forceinline__ void settle(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kWaitTimeoutNs / 4) {
    }
}

template <int BM, int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm1(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, const G1Params p) {
    using L = G1Layout<BM>;
    // This CTA's output-channel block and row slot; tiles slot, slot + nslots, ...
    const int cblk = (int)(blockIdx.x % (unsigned)p.cblocks);
    const int64_t slot = blockIdx.x / p.cblocks, nslots = gridDim.x / p.cblocks;
    const int64_t tiles = (p.n + kRows - 1) / kRows;
    const int64_t my_tiles = slot < tiles ? (tiles - 1 - slot) / nslots + 1 : 0;
    if (my_tiles == 0) return;  // the whole CTA, before any barrier or tensor memory

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int wch = p.cin / kChunk, S = p.stages;
    uint8_t* w_s = smem;
    uint8_t* x_ring = w_s + wch * L::kWChunkBytes;
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(x_ring + S * kXStageBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stage) + L::kStgBytes);
    int* misc = reinterpret_cast<int*>(bars + L::num_bars(wch, S));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
    volatile int* abort_flag = misc + 1;
    const uint32_t wF0 = smem_addr(bars), xF0 = wF0 + 8 * wch, xE0 = xF0 + 8 * S;
    const uint32_t accF0 = xE0 + 8 * S, accE0 = accF0 + 8 * kAccBufs, drain = accE0 + 8 * kAccBufs;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == kWarpTma * 32) {
        for (int c = 0; c < wch; ++c) mbar_init(wF0 + 8 * c, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(xF0 + 8 * s, 1);
            mbar_init(xE0 + 8 * s, 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(accF0 + 8 * b, 1);
            mbar_init(accE0 + 8 * b, kEpiWarps);
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
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, kRows);
            int64_t q = 0;  // x stages consumed
            for (int64_t it = 0; it < my_tiles && !aborted; ++it) {
                const int buf = (int)(it % kAccBufs);
                if (it >= kAccBufs) {  // the epilogue has read this accumulator's previous tile
                    if (!wait_bar<0>(accE0 + 8 * buf, (uint32_t)((it / kAccBufs - 1) & 1), abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                }
                const uint32_t d = tmem + (uint32_t)(buf * kRows);
                for (int c = 0; c < wch; ++c, ++q) {
                    if (it == 0 && !wait_bar<0>(wF0 + 8 * c, 0, abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    const int s = (int)(q % S);
                    if (!wait_bar<0>(xF0 + 8 * s, (uint32_t)((q / S) & 1), abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    // A: the weight chunk, MN-major (64-channel boxes 8 KB apart); B: the
                    // x stage, K-major, 128 rows of 128 bytes.  K steps of 16 channels
                    // advance the start address (>> 4) by 2048 and 32 bytes.
                    const uint64_t adesc0 = smem_desc(smem_addr(w_s + c * L::kWChunkBytes), kChunk * 128, 1024, 2);
                    const uint64_t bdesc0 = smem_desc(smem_addr(x_ring + s * kXStageBytes), 16, 1024, 2);
#pragma unroll
                    for (int kk = 0; kk < kChunk / 16; ++kk)
                        mma_bf16(d, adesc0 + (uint64_t)((kk * 2048) >> 4), bdesc0 + (uint64_t)((kk * 32) >> 4), idesc,
                                 (c > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(xE0 + 8 * s);  // the stage is free once these MMAs have read it
                }
                if (aborted) break;
                mma_commit(accF0 + 8 * buf);
            }
            if (aborted) {
                mma_commit(drain);  // wait for the MMAs in flight before TMEM is freed
                settle(drain, 0);
            }
        }
        __syncwarp();
    } else if (warp == kWarpTma) {
        // ------------------------------------------------ TMA producer (lane 0)
        if (lane == 0) {
            for (int c = 0; c < wch; ++c) {
                mbar_arrive_expect_tx(wF0 + 8 * c, L::kWChunkBytes);
#pragma unroll
                for (int a = 0; a < BM / 64; ++a)
                    tma_load_2d(smem_addr(w_s + c * L::kWChunkBytes + a * kChunk * 128), &wmap, cblk * BM + a * 64,
                                c * kChunk, wF0 + 8 * c);
            }
            int64_t q = 0;  // x stages issued
            for (int64_t it = 0; it < my_tiles && !aborted; ++it) {
                // rows past n read as zeros (their columns are not stored)
                const int row0 = (int)((slot + it * nslots) * kRows);
                for (int c = 0; c < wch; ++c, ++q) {
                    const int s = (int)(q % S);
                    if (q >= S && !wait_bar<0>(xE0 + 8 * s, (uint32_t)((q / S - 1) & 1), abort_flag, p.err)) {
                        aborted = true;
                        break;
                    }
                    mbar_arrive_expect_tx(xF0 + 8 * s, kXStageBytes);
                    tma_load_2d(smem_addr(x_ring + s * kXStageBytes), &xmap, c * kChunk, row0, xF0 + 8 * s);
                }
            }
            if (aborted) {
                // the weight chunks and the last S stages issued land before the CTA exits
                for (int c = 0; c < wch; ++c) settle(wF0 + 8 * c, 0);
                for (int64_t qi = q > S ? q - S : 0; qi < q; ++qi)
                    settle(xF0 + 8 * (int)(qi % S), (uint32_t)((qi / S) & 1));
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int half = (warp - kWarpEpi0) >> 2;  // this warp's 32-column chunks: half, half + 2
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        __nv_bfloat16* stg = stage + (warp - kWarpEpi0) * L::kStageRows * L::kChPerWarp;
        const bool lane_ok = lane < L::kChPerWarp;
        const int ch_base = cblk * BM + quarter * L::kChPerWarp;
        const float bv = (p.bias && lane_ok) ? __bfloat162float(p.bias[ch_base + lane]) : 0.0f;
        const tc::EpiOut eo{p.out, p.residual, p.cout, p.act};
        float s1 = 0.0f, s2 = 0.0f;  // this lane's channel statistics over all its tiles (fused epilogue)
        for (int64_t it = 0; it < my_tiles; ++it) {
            const int buf = (int)(it % kAccBufs);
            const int64_t row_t0 = (slot + it * nslots) * kRows;
            const int t_eff = (int)min((int64_t)kRows, p.n - row_t0);
            int orow[kChunksPerWarp];
#pragma unroll
            for (int c4 = 0; c4 < kChunksPerWarp; ++c4) {
                const int col = (half + 2 * c4) * 32 + lane;
                orow[c4] = col < t_eff ? (int)(row_t0 + col) : -1;
            }
            if constexpr (kEpi != kEpiPlain) {
                if (p.residual) {
#pragma unroll
                    for (int c4 = 0; c4 < kChunksPerWarp; ++c4)
                        if (orow[c4] >= 0) prefetch_l2(p.residual + (int64_t)orow[c4] * p.cout + ch_base);
                }
            }
            if (!warp_wait_bar<kSleepEpilogue>(accF0 + 8 * buf, (uint32_t)((it / kAccBufs) & 1), abort_flag,
                                               p.err)) {
                aborted = true;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c4 = 0; c4 < kChunksPerWarp; ++c4) {
                const int cc = half + 2 * c4;
                if (cc * 32 < t_eff) {
                    float v[32];
                    tmem_ld_x32(tmem + lane_base + (uint32_t)(buf * kRows + cc * 32), v);
                    tmem_wait_ld();
                    tc::store_chunk<kEpi, L::kChPerWarp, L::kStageRows>(v, orow[c4], lane, lane_ok, bv, ch_base,
                                                                        cc * 32, t_eff, eo, stg, s1, s2);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accE0 + 8 * buf);
        }
        if constexpr (kEpi != kEpiPlain) {
            if (!aborted && p.stats && lane_ok) {
                atomicAdd(p.stats + ch_base + lane, s1);
                atomicAdd(p.stats + p.cout + ch_base + lane, s2);
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

int g_force_stages = 0;  // test hook: x stages (0 = as many as fit)

template <int BM>
spconv_status_t launch(const MapData& m, const void* x, int cin, const void* w, const void* bias, void* out,
                       int cout, const Epilogue& epi, cudaStream_t stream, cudaError_t* ce) {
    using L = G1Layout<BM>;
    int stages = 0;
    if (g_force_stages > 0) {
        stages = g_force_stages < kMaxStages ? g_force_stages : kMaxStages;
        while (stages > kMinStages && L::smem_bytes(cin, stages) > kMaxSmem) --stages;
    } else {
        stages = kMaxStages;
        while (stages > kMinStages && L::smem_bytes(cin, stages) > kMaxSmem) --stages;
    }
    if (L::smem_bytes(cin, stages) > kMaxSmem) return SPCONV_ERR_UNSUPPORTED;
    tc::EncodeTiledFn enc = tc::encode_fn();
    if (!enc) {
        *ce = cudaErrorSymbolNotFound;
        return SPCONV_ERR_CUDA;
    }
    const int cblocks = cout / BM;
    // Weights [cin, cout]: boxes of 64 output channels (128 B, 128-byte swizzle)
    // by 64 input channels.  Features [n, cin]: boxes of 64 channels by 128 rows,
    // swizzled the same way; n >= kRows, so a box is never taller than the tensor.
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap wmap, xmap;
    const cuuint64_t wdims[2] = {(cuuint64_t)cout, (cuuint64_t)cin};
    const cuuint64_t wstrides[1] = {(cuuint64_t)cout * 2};
    const cuuint32_t wbox[2] = {64, (cuuint32_t)kChunk};
    CUresult r = enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), wdims, wstrides, wbox, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    const cuuint64_t xdims[2] = {(cuuint64_t)cin, (cuuint64_t)m.n};
    const cuuint64_t xstrides[1] = {(cuuint64_t)cin * 2};
    const cuuint32_t xbox[2] = {(cuuint32_t)kChunk, (cuuint32_t)kRows};
    if (r == CUDA_SUCCESS)
        r = enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), xdims, xstrides, xbox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *ce = cudaErrorInvalidValue;
        return SPCONV_ERR_CUDA;
    }
    int dev = 0;
    cudaError_t de = cudaGetDevice(&dev);
    if (de != cudaSuccess) {
        *ce = de;
        return SPCONV_ERR_CUDA;
    }
    const int kind = tc::epi_kind(epi);
    auto kernel = kind == kEpiPlain  ? k_gemm1<BM, kEpiPlain>
                  : kind == kEpiRelu ? k_gemm1<BM, kEpiRelu>
                  : kind == kEpiSilu ? k_gemm1<BM, kEpiSilu>
                                     : k_gemm1<BM, kEpiGelu>;
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
    G1Params p;
    p.n = m.n;
    p.cin = cin;
    p.cout = cout;
    p.cblocks = cblocks;
    p.stages = stages;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.act = epi.act;
    p.residual = static_cast<const __nv_bfloat16*>(epi.residual);
    p.stats = epi.stats;
    p.err = m.fwd_err;
    // One CTA per SM: row slots of cblocks CTAs each, at most one slot per tile.
    const int64_t tiles = (m.n + kRows - 1) / kRows;
    int64_t nslots = m.num_sms / cblocks;
    if (nslots < 1) nslots = 1;
    if (nslots > tiles) nslots = tiles;
    kernel<<<(unsigned)(nslots * cblocks), kThreads, L::smem_bytes(cin, stages), stream>>>(wmap, xmap, p);
    *ce = cudaGetLastError();
    return *ce == cudaSuccess ? SPCONV_OK : SPCONV_ERR_CUDA;
}

}  // namespace

void set_forced_gemm1_stages(int stages) { g_force_stages = stages; }

spconv_status_t launch_forward_gemm1(const MapData& m, const void* x, int cin, const void* w, const void* bias,
                                     void* out, int cout, const Epilogue& epi, cudaStream_t stream, cudaError_t* ce) {
    *ce = cudaSuccess;
    if (m.kernel_size != 1 || cin % kChunk != 0 || cin / kChunk > kMaxWChunks || cout % 64 != 0 || m.n < kRows)
        return SPCONV_ERR_UNSUPPORTED;
    if (cout % 128 == 0) return launch<128>(m, x, cin, w, bias, out, cout, epi, stream, ce);
    return launch<64>(m, x, cin, w, bias, out, cout, epi, stream, ce);
}

}  // namespace spconv
