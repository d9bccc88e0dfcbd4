// Pieces shared by the tcgen05 forward kernels (forward_win.cu, forward_gemm1.cu):
// the bounded barrier waits and the epilogue store of one 32-column accumulator
// chunk.  Both kernels hold D transposed in tensor memory (lane = output channel,
// column = output row), so the epilogue code is the same.
#pragma once

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace spconv {
namespace tc {

using namespace sm100;

constexpr uint64_t kWaitTimeoutNs = 4000000000ull;

// Kernel instantiations by epilogue: the plain store, and the fused epilogue with
// ReLU or none (chosen at run time), SiLU or GELU, so no instantiation carries the
// code of the activations it does not run.
constexpr int kEpiPlain = 0, kEpiRelu = 1, kEpiSilu = 2, kEpiGelu = 3;

inline int epi_kind(const Epilogue& epi) {
    const bool fused = epi.act != SPCONV_ACT_NONE || epi.residual != nullptr || epi.stats != nullptr;
    if (!fused) return kEpiPlain;
    return epi.act == SPCONV_ACT_SILU ? kEpiSilu : (epi.act == SPCONV_ACT_GELU ? kEpiGelu : kEpiRelu);
}

// A waiting thread polls the barrier; while the phase is not complete it may back
// off with __nanosleep, doubling the pause up to kMaxSleepNs.  After
// kWaitTimeoutNs it sets the CTA's abort flag, records kFwdErrTimeout and returns
// false; a wait that sees the abort flag set returns false too.
template <uint32_t kMaxSleepNs>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = 0;
    uint32_t pause = 32;
    for (uint32_t i = 1;; ++i) {
        if constexpr (kMaxSleepNs > 0) {
            __nanosleep(pause);
            pause = pause < kMaxSleepNs ? 2 * pause : pause;
        }
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) != 0) continue;  // the timer and the abort flag every few polls
        if (*abort_flag) return false;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            atomicOr(err, kFwdErrTimeout);
            return false;
        }
    }
}

// Lane 0 waits; the warp learns the outcome.
template <uint32_t kMaxSleepNs>
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* err) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = wait_bar<kMaxSleepNs>(bar, parity, abort_flag, err) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda); null if the driver does not provide it.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

// Where an epilogue warp's results go.
struct EpiOut {
    __nv_bfloat16* out;
    const __nv_bfloat16* residual;  // [n, cout] added after the activation, or null
    int cout;
    int act;                        // spconv_act_t (kEpiRelu instantiation: none or ReLU)
};

// Stores one 32-column accumulator chunk of an epilogue warp.  Lane l holds v[j],
// the accumulator of output channel ch_base + l (lanes >= kChPerWarp hold none)
// and chunk column j; `orow` (lane j's value) is the output row of column j, or
// -1 past the tile's rows.  Rows pass through the warp's staging buffer stg
// (kStageRows rows of kChPerWarp channels) so every store is 16 bytes wide and
// each output row slice is written once.  The fused instantiations apply
// act(v + bias), add the residual element and add the stored (rounded) values of
// the columns below t_eff to s1 and their squares to s2.
template <int kEpi, int kChPerWarp, int kStageRows>
__device__ __forceinline__ void store_chunk(const float (&v)[32], int orow, int lane, bool lane_ok, float bv,
                                            int ch_base, int col0, int t_eff, const EpiOut& eo,
                                            __nv_bfloat16* stg, float& s1, float& s2) {
    constexpr int kVecPerRow = kChPerWarp * 2 / 16;
#pragma unroll
    for (int hp = 0; hp < 32 / kStageRows; ++hp) {
        if constexpr (kEpi == kEpiPlain) {
            if (lane_ok) {
#pragma unroll
                for (int e = 0; e < kStageRows; ++e)
                    stg[e * kChPerWarp + lane] = __float2bfloat16_rn(v[hp * kStageRows + e] + bv);
            }
        } else {
            // fused epilogue: act(conv + bias) (+ residual) in fp32, then the
            // rounded value is stored and counted in the statistics
            const int c0 = col0 + hp * kStageRows;  // chunk column of row e = c0 + e
            float rv[kStageRows];                   // residual elements (0 when there is none)
            if (eo.residual) {
                // the output rows of these columns, then their residual elements,
                // loaded together (a missing row reads row 0)
                int ro[kStageRows];
#pragma unroll
                for (int e = 0; e < kStageRows; ++e) ro[e] = __shfl_sync(0xffffffffu, orow, hp * kStageRows + e);
#pragma unroll
                for (int e = 0; e < kStageRows; ++e)
                    rv[e] = lane_ok ? __bfloat162float(
                                          eo.residual[(int64_t)(ro[e] > 0 ? ro[e] : 0) * eo.cout + ch_base + lane])
                                    : 0.0f;
            } else {
#pragma unroll
                for (int e = 0; e < kStageRows; ++e) rv[e] = 0.0f;
            }
            if (lane_ok) {
#pragma unroll
                for (int e = 0; e < kStageRows; ++e) {
                    float y = v[hp * kStageRows + e] + bv;
                    if constexpr (kEpi == kEpiRelu) {
                        if (eo.act == SPCONV_ACT_RELU) y = fmaxf(y, 0.0f);
                    } else if constexpr (kEpi == kEpiSilu) {
                        // fast exponential and division: their error is far below the
                        // bf16 rounding of out (a huge denominator gives -0 for y << 0)
                        y = __fdividef(y, 1.0f + __expf(-y));
                    } else {
                        y = epi_act(SPCONV_ACT_GELU, y);
                    }
                    const __nv_bfloat16 q = __float2bfloat16_rn(y + rv[e]);
                    stg[e * kChPerWarp + lane] = q;
                    if (c0 + e < t_eff) {
                        const float f = __bfloat162float(q);
                        s1 += f;
                        s2 += f * f;
                    }
                }
            }
        }
        __syncwarp();
#pragma unroll
        for (int e = lane; e < kStageRows * kVecPerRow; e += 32) {
            const int row = e / kVecPerRow, vq = e % kVecPerRow;
            const int o = __shfl_sync(0xffffffffu, orow, hp * kStageRows + row);
            if (o >= 0) {
                const int4 val = *reinterpret_cast<const int4*>(stg + row * kChPerWarp + vq * 8);
                *reinterpret_cast<int4*>(eo.out + (int64_t)o * eo.cout + ch_base + vq * 8) = val;
            }
        }
        __syncwarp();
    }
}

}  // namespace tc
}  // namespace spconv
