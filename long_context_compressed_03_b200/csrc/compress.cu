// compress.cu -- stage 1: overlapping mean-pool compression + projection.
//
// out[b, i, :] = (mean_{p in win(i)} x[b, p, :]) @ W
//   overlap: win(i) = [m(i-1), m(i+1)) ∩ [0, n)  -- own block + previous block
//   plain:   win(i) = [m i, m(i+1))
// ("百万上下文从「奢侈品」变「日用品」…" §3.2 mean pool + projection;
//  "DS-V4 分析&学习" §1.3 2m-position overlap; "DeepSeek V4 CSA + CP 迁移到 HP…"
//  §3.2 ratio 4 overlapping, ratio 128 not.)
//
// One CTA owns a tile of ET consecutive entries of one batch element.  It
// streams the tile's blocks once (each block's m rows summed in fp32, rows
// read coalesced along the feature dimension), forms the pooled rows from
// one or two block sums, multiplies them by W (fp32 FMA, W read through L2)
// and writes the tile in the requested format; the fp8 epilogue reduces each
// row's amax across a warp and quantises it in place.
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;  // entries per CTA

template <typename Tin, int OUT>
__global__ void __launch_bounds__(kThreads) compress_kernel(CompressArgs a) {
    extern __shared__ float smem[];
    const int d_in = a.d_in, d_out = a.d_out, m = a.m, n = a.n, N_c = a.N_c;
    const int b = blockIdx.y;
    const int i0 = blockIdx.x * kTile;
    const int ne = min(kTile, N_c - i0);
    float* bsum = smem;                           // [kTile + 1][d_in]: blocks i0-1 .. i0+kTile-1
    float* pooled = bsum + (kTile + 1) * d_in;    // [kTile][d_in]
    float* outs = pooled + kTile * d_in;          // [kTile][d_out]
    const Tin* x = static_cast<const Tin*>(a.x) + (size_t)b * n * d_in;
    const Tin* W = static_cast<const Tin*>(a.W);

    // block sums of blocks jb = i0-1+jj (jj = 0 .. ne)
    for (int p = threadIdx.x; p < (ne + 1) * d_in; p += kThreads) {
        const int jj = p / d_in, c = p - jj * d_in;
        const int jb = i0 - 1 + jj;
        float acc = 0.0f;
        if (jb >= 0 && (a.overlap || jj > 0)) {
            const Tin* src = x + (size_t)jb * m * d_in + c;
            for (int r = 0; r < m; ++r) acc += to_f32(src[(size_t)r * d_in]);
        }
        bsum[p] = acc;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < ne * d_in; p += kThreads) {
        const int e = p / d_in, c = p - e * d_in;
        const int i = i0 + e;
        const int lo = a.overlap ? max(0, m * (i - 1)) : m * i;
        const float cnt = (float)(m * (i + 1) - lo);
        const float s = bsum[(e + 1) * d_in + c] + (a.overlap ? bsum[e * d_in + c] : 0.0f);
        pooled[p] = s / cnt;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < ne * d_out; p += kThreads) {
        const int e = p / d_out, o = p - e * d_out;
        const float* pr = pooled + e * d_in;
        float acc = 0.0f;
        for (int c = 0; c < d_in; ++c) acc = fmaf(pr[c], to_f32(W[(size_t)c * d_out + o]), acc);
        outs[p] = acc;
    }
    __syncthreads();

    const size_t row0 = (size_t)b * N_c + i0;
    if constexpr (OUT == DT_E4M3) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        uint8_t* out = static_cast<uint8_t*>(a.out);
        for (int e = warp; e < ne; e += kThreads / 32) {
            float amax = 0.0f;
            for (int o = lane; o < d_out; o += 32) amax = fmaxf(amax, fabsf(outs[e * d_out + o]));
            for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
            for (int o = lane; o < d_out; o += 32)
                out[(row0 + e) * d_out + o] = e4m3_code(__fdiv_rn(outs[e * d_out + o], scale));
            if (lane == 0) a.out_row_scale[row0 + e] = scale;
        }
    } else {
        using Tout = typename std::conditional<OUT == DT_F32, float, __nv_bfloat16>::type;
        Tout* out = static_cast<Tout*>(a.out);
        for (int p = threadIdx.x; p < ne * d_out; p += kThreads)
            store_out<Tout>(out + row0 * d_out + p, outs[p]);
    }
}

template <typename Tin, int OUT>
cudaError_t launch_t(const CompressArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)(2 * kTile + 1) * a.d_in + (size_t)kTile * a.d_out);
    auto kern = compress_kernel<Tin, OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.N_c + kTile - 1) / kTile, a.B);
    kern<<<grid, kThreads, smem, s>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s, const char** why) {
    if (a.N_c <= 0 || a.B <= 0) return cudaSuccess;
    if (a.x_dt == DT_F32) {
        if (a.out_dt == DT_F32) return launch_t<float, DT_F32>(a, s);
        if (a.out_dt == DT_BF16) return launch_t<float, DT_BF16>(a, s);
        if (a.out_dt == DT_E4M3) return launch_t<float, DT_E4M3>(a, s);
    } else if (a.x_dt == DT_BF16) {
        if (a.out_dt == DT_BF16) return launch_t<__nv_bfloat16, DT_BF16>(a, s);
        if (a.out_dt == DT_E4M3) return launch_t<__nv_bfloat16, DT_E4M3>(a, s);
    }
    *why = "csa_compress: unsupported (x_dt, out_dt) pair";
    return cudaErrorNotSupported;
}

}  // namespace csa
