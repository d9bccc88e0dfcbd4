// CUDA-core forward: one thread per (output row, output channel), fp32
// accumulation over the active offsets and input channels.  It serves the fp32
// path (any channel count) and, for bf16, as an independent GPU cross-check of
// the tensor-core kernel.
#include "common.cuh"

namespace spconv {
namespace {

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
// Stores v in the output type and returns the stored value.
__device__ __forceinline__ float store(float* p, float v) {
    *p = v;
    return v;
}
__device__ __forceinline__ float store(__nv_bfloat16* p, float v) {
    const __nv_bfloat16 q = __float2bfloat16_rn(v);
    *p = q;
    return __bfloat162float(q);
}

constexpr int kRowsPerBlock = 8;

// grid: (ceil(n / kRowsPerBlock), ceil(cout / blockDim.x)).
template <typename T>
__global__ void k_forward_simt(const int32_t* __restrict__ nbr, int64_t n, int kvol, const T* __restrict__ x,
                               int cin, const T* __restrict__ w, const T* __restrict__ bias, T* out, int cout,
                               int act, const T* residual, float* __restrict__ stats) {
    // out and residual may be the same array (each element is read, then written,
    // by one thread), so neither is __restrict__
    const int co = blockIdx.y * blockDim.x + threadIdx.x;
    const int64_t row0 = (int64_t)blockIdx.x * kRowsPerBlock;
    float s1 = 0.0f, s2 = 0.0f;  // this thread's share of the channel statistics
    for (int r = 0; r < kRowsPerBlock; ++r) {
        const int64_t row = row0 + r;
        if (row >= n || co >= cout) break;
        float acc = bias ? to_f(bias[co]) : 0.0f;
        for (int k = 0; k < kvol; ++k) {
            const int64_t j = (kvol == 1) ? row : (int64_t)nbr[row * kvol + k];
            if (j < 0) continue;
            const T* xj = x + j * cin;
            const T* wk = w + (int64_t)k * cin * cout + co;
            for (int ci = 0; ci < cin; ++ci) acc = fmaf(to_f(xj[ci]), to_f(wk[(int64_t)ci * cout]), acc);
        }
        float y = epi_act(act, acc);
        if (residual) y += to_f(residual[row * cout + co]);
        const float q = store(out + row * cout + co, y);
        s1 += q;
        s2 += q * q;
    }
    if (stats && co < cout && row0 < n) {
        atomicAdd(stats + co, s1);
        atomicAdd(stats + cout + co, s2);
    }
}

}  // namespace

cudaError_t launch_forward_simt(const MapData& m, spconv_dtype_t dtype, const void* x, int cin, const void* w,
                                const void* bias, void* out, int cout, const Epilogue& epi, cudaStream_t stream) {
    if (m.n == 0) return cudaSuccess;
    const int kvol = m.kernel_size == 3 ? kVol3 : 1;
    const int threads = cout >= 128 ? 128 : ((cout + 31) / 32) * 32;
    dim3 grid((unsigned)((m.n + kRowsPerBlock - 1) / kRowsPerBlock), (unsigned)((cout + threads - 1) / threads));
    if (dtype == SPCONV_F32) {
        k_forward_simt<float><<<grid, threads, 0, stream>>>(m.nbr, m.n, kvol, (const float*)x, cin,
                                                            (const float*)w, (const float*)bias, (float*)out,
                                                            cout, epi.act, (const float*)epi.residual, epi.stats);
    } else {
        k_forward_simt<__nv_bfloat16><<<grid, threads, 0, stream>>>(
            m.nbr, m.n, kvol, (const __nv_bfloat16*)x, cin, (const __nv_bfloat16*)w, (const __nv_bfloat16*)bias,
            (__nv_bfloat16*)out, cout, epi.act, (const __nv_bfloat16*)epi.residual, epi.stats);
    }
    return cudaGetLastError();
}

}  // namespace spconv
