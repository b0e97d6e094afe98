// compress_append.cu -- decode-time stage 1: one new token per batch element
// updates the compressor state; a token that completes block j writes entry j.
//
//   state[b] = (sum of the last complete block, running sum of the current one)
//   cache[b, j] = (mean over blocks j-1 and j if overlap and j > 0, else over
//                  block j) @ W      when the token at pos[b] completes block j
// ("DS-V4 分析&学习", opening summary: compressed cache + state cache + tail
//  state; §1.3: overlapping entries span the previous and the current block.)
//
// One CTA per batch element: the state update is a d_in-wide vector add, the
// completed entry a d_in x d_out product with W read through L2 (fp32 FMA,
// pooled row staged in shared memory), and the E4M3 epilogue reduces the
// row's amax across the CTA (after one warp rotates the row, for the
// Hadamard type).  The work per step is a few KB: the launch is
// bound by latency, not bandwidth.
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;

template <typename Tin, int OUT>
__global__ void __launch_bounds__(kThreads) compress_append_kernel(AppendArgs a) {
    __shared__ float pooled[256];
    __shared__ float outs[256];
    __shared__ float red[kThreads / 32];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int p = a.pos[b];
    if (p < 0) return;                                  // no token for this element
    const int d_in = a.d_in, d_out = a.d_out, m = a.m;
    const bool complete = (p + 1) % m == 0;
    const int j = p / m;
    const bool both = a.overlap && j > 0;
    const float cnt = both ? (float)(2 * m) : (float)m;
    float* prev = a.state + (size_t)b * 2 * d_in;
    float* cur = prev + d_in;
    const Tin* x = static_cast<const Tin*>(a.x) + (size_t)b * d_in;
    for (int c = tid; c < d_in; c += kThreads) {
        const float v = cur[c] + to_f32(x[c]);
        if (complete) {
            pooled[c] = ((both ? prev[c] : 0.0f) + v) / cnt;
            prev[c] = v;
            cur[c] = 0.0f;
        } else {
            cur[c] = v;
        }
    }
    if (!complete || j >= a.N_cap) return;              // uniform across the CTA
    const long crow = cache_row(a.pages, a.N_cap, b, j);
    if (crow < 0) return;                               // page outside the pool: not written
    __syncthreads();
    const Tin* W = static_cast<const Tin*>(a.W);
    for (int o = tid; o < d_out; o += kThreads) {
        float acc = 0.0f;
        for (int c = 0; c < d_in; ++c) acc = fmaf(pooled[c], to_f32(W[(size_t)c * d_out + o]), acc);
        outs[o] = acc;
    }
    __syncthreads();
    const size_t row = (size_t)crow;
    if constexpr (OUT == DT_E4M3 || OUT == DT_E4M3H) {
        if constexpr (OUT == DT_E4M3H) {
            if (tid < 32) hadamard_row_warp(outs, d_out, a.hnorm);
            __syncthreads();
        }
        float amax = 0.0f;
        for (int o = tid; o < d_out; o += kThreads) amax = fmaxf(amax, fabsf(outs[o]));
        for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if ((tid & 31) == 0) red[tid >> 5] = amax;
        __syncthreads();
        amax = 0.0f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
        const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint8_t* out = static_cast<uint8_t*>(a.cache) + row * d_out;
        for (int o = tid; o < d_out; o += kThreads) out[o] = e4m3_code(__fdiv_rn(outs[o], scale));
        if (tid == 0) a.cache_scale[row] = scale;
    } else {
        using Tout = typename std::conditional<OUT == DT_F32, float, __nv_bfloat16>::type;
        Tout* out = static_cast<Tout*>(a.cache) + row * d_out;
        for (int o = tid; o < d_out; o += kThreads) store_out<Tout>(out + o, outs[o]);
    }
    if (tid == 0 && a.n_entries) a.n_entries[b] = j + 1;
}

template <typename Tin, int OUT>
cudaError_t launch_t(const AppendArgs& a, cudaStream_t s) {
    compress_append_kernel<Tin, OUT><<<(unsigned)a.B, kThreads, 0, s>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress_append(const AppendArgs& a, cudaStream_t s, const char** why) {
    if (a.B <= 0) return cudaSuccess;
    if (a.x_dt == DT_F32) {
        if (a.out_dt == DT_F32) return launch_t<float, DT_F32>(a, s);
        if (a.out_dt == DT_BF16) return launch_t<float, DT_BF16>(a, s);
        if (a.out_dt == DT_E4M3) return launch_t<float, DT_E4M3>(a, s);
        if (a.out_dt == DT_E4M3H) return launch_t<float, DT_E4M3H>(a, s);
    } else if (a.x_dt == DT_BF16) {
        if (a.out_dt == DT_BF16) return launch_t<__nv_bfloat16, DT_BF16>(a, s);
        if (a.out_dt == DT_E4M3) return launch_t<__nv_bfloat16, DT_E4M3>(a, s);
        if (a.out_dt == DT_E4M3H) return launch_t<__nv_bfloat16, DT_E4M3H>(a, s);
    }
    *why = "csa_compress_append: unsupported (x_dt, out_dt) pair";
    return cudaErrorNotSupported;
}

}  // namespace csa
