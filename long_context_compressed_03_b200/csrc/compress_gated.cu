// compress_gated.cu -- stage 1, learned variant: the gated-softmax compressor.
//
//   v_p = x_p @ W_kv,   z_p = x_p @ W_gate + ape[p mod m]   (c * d_out values;
//                                                           c = 2 if overlapping)
//   out[i, e] = sum softmax(z) v over the terms of entry i's window, per channel:
//     overlapping: block i-1 through channel e, block i through channel d_out + e
//     plain:       block i through channel e
// ("DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" §3.2: linear_wkv +
//  linear_wgate + softmax / split / reshape, the APE parameter, ratio 4
//  overlapping and ratio 128 not.)
//
// One CTA owns TE consecutive entries of one batch element (TE = 64/m minus
// one when overlapping, at least 1) and the positions they read.  It walks
// the output channels in slices of 32.  For a slice it projects 64 positions
// at a time onto the slice's columns of [W_kv | W_gate] (both halves when
// overlapping): a register-tiled fp32 product, x rows and 32-row chunks of
// the weights staged in shared memory.  Each thread then folds its
// (entry, channel) pairs' terms into an online softmax held in registers, so
// a window may span several 64-position steps (ratio 128).  The pooled rows
// go through the entry epilogue shared with the mean-pool compressor.
#include <math.h>

#include "common.cuh"
#include "entry_epilogue.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 64;                            // positions projected per step
constexpr int kDC = 32;                              // output channels per slice
constexpr int kKC = 32;                              // weight rows staged per step
constexpr int kMaxPairs = 64 * kDC / kThreads;       // (entry, channel) pairs per thread

__host__ __device__ inline int tile_entries(int m, int overlap) {
    const int t = 64 / m - overlap;
    return t < 1 ? 1 : t;
}

template <typename Tin, int OUT>
__global__ void __launch_bounds__(kThreads) compress_gated_kernel(GatedArgs a) {
    extern __shared__ float smem[];
    const int d_in = a.d_in, d_out = a.d_out, m = a.m, ov = a.overlap;
    const int cw = ov ? 2 * d_out : d_out;           // projected width
    const int nh = ov ? 2 : 1;                       // channel halves
    const int ncols = 2 * nh * kDC;                  // [kv halves][gate halves] x 32
    const int TE = tile_entries(m, ov);
    const int b = blockIdx.y;
    const int i0 = blockIdx.x * TE;
    const int ne = min(TE, a.N_c - i0);
    const int p_lo = max(0, m * (i0 - ov));          // first position the tile reads
    const int p_hi = m * (i0 + ne);                  // one past the last
    float* xs = smem;                                // [kRows][d_in]
    float* ws = xs + kRows * d_in;                   // [kKC][128]
    float* proj = ws + kKC * 128;                    // [kRows][128]
    float* outs = proj + kRows * 128;                // [TE][d_out]
    const Tin* x = static_cast<const Tin*>(a.x) + (size_t)b * a.n * d_in;
    const Tin* Wkv = static_cast<const Tin*>(a.W_kv);
    const Tin* Wg = static_cast<const Tin*>(a.W_gate);
    const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;

    for (int e0 = 0; e0 < d_out; e0 += kDC) {
        const int dc = min(kDC, d_out - e0);         // 32, or 16 for the last slice
        float zmax[kMaxPairs], den[kMaxPairs], num[kMaxPairs];
#pragma unroll
        for (int s = 0; s < kMaxPairs; ++s) {
            zmax[s] = -INFINITY;
            den[s] = 0.0f;
            num[s] = 0.0f;
        }
        for (int r0 = p_lo; r0 < p_hi; r0 += kRows) {
            const int nr = min(kRows, p_hi - r0);
            __syncthreads();                         // xs / proj of the previous step consumed
            for (int q = tid; q < kRows * d_in; q += kThreads) {
                const int r = q / d_in, k = q - r * d_in;
                xs[q] = r < nr ? to_f32(x[(size_t)(r0 + r) * d_in + k]) : 0.0f;
            }
            // ---- projection: rows 8 ty .. +7, columns 4 tx .. +3 of the slice
            float acc[8][4];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.0f;
            for (int k0 = 0; k0 < d_in; k0 += kKC) {
                const int kc = min(kKC, d_in - k0);
                __syncthreads();                     // xs written / previous chunk consumed
                for (int q = tid; q < kc * ncols; q += kThreads) {
                    const int kr = q / ncols, j = q - kr * ncols;
                    const int grp = j / kDC, ec = j - grp * kDC;
                    const bool gate = grp >= nh;
                    const int half = gate ? grp - nh : grp;
                    float w = 0.0f;
                    if (ec < dc) w = to_f32((gate ? Wg : Wkv)[(size_t)(k0 + kr) * cw + half * d_out + e0 + ec]);
                    ws[kr * 128 + j] = w;
                }
                __syncthreads();
                if (4 * tx < ncols) {
#pragma unroll 4
                    for (int kk = 0; kk < kc; ++kk) {
                        const float4 w4 = *reinterpret_cast<const float4*>(ws + kk * 128 + 4 * tx);
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            const float xv = xs[(8 * ty + r) * d_in + k0 + kk];
                            acc[r][0] = fmaf(xv, w4.x, acc[r][0]);
                            acc[r][1] = fmaf(xv, w4.y, acc[r][1]);
                            acc[r][2] = fmaf(xv, w4.z, acc[r][2]);
                            acc[r][3] = fmaf(xv, w4.w, acc[r][3]);
                        }
                    }
                }
            }
            if (4 * tx < ncols) {
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    *reinterpret_cast<float4*>(proj + (8 * ty + r) * 128 + 4 * tx) =
                        make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
            }
            __syncthreads();
            // ---- online softmax of this step's terms, per owned (entry, channel)
#pragma unroll
            for (int s = 0; s < kMaxPairs; ++s) {
                const int q = tid + s * kThreads;
                const int te = q / kDC, ec = q - te * kDC;
                if (te < ne && ec < dc) {
                    const int i = i0 + te;
                    for (int h = 0; h < nh; ++h) {
                        const int blk = ov ? i - 1 + h : i;  // the block read through half h
                        if (blk < 0) continue;
                        const int lo = max(blk * m, r0), hi = min(blk * m + m, r0 + nr);
                        const int kvc = h * kDC + ec, gc = (nh + h) * kDC + ec;
                        const float* ap = a.ape + (size_t)h * d_out + e0 + ec;
                        for (int p = lo; p < hi; ++p) {
                            const int r = p - r0;
                            const float z = proj[r * 128 + gc] + ap[(size_t)(p % m) * cw];
                            const float v = proj[r * 128 + kvc];
                            if (z > zmax[s]) {
                                const float f = expf(zmax[s] - z);   // 0 for the first term
                                den[s] *= f;
                                num[s] *= f;
                                zmax[s] = z;
                            }
                            const float w = expf(z - zmax[s]);
                            den[s] += w;
                            num[s] = fmaf(w, v, num[s]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int s = 0; s < kMaxPairs; ++s) {
            const int q = tid + s * kThreads;
            const int te = q / kDC, ec = q - te * kDC;
            if (te < ne && ec < dc) outs[te * d_out + e0 + ec] = num[s] / den[s];
        }
    }
    __syncthreads();
    store_entry_rows<OUT, kThreads>(outs, ne, d_out, a.out, a.out_row_scale, (size_t)b * a.N_c + i0,
                                    a.hnorm);
}

template <typename Tin, int OUT>
cudaError_t launch_t(const GatedArgs& a, cudaStream_t s) {
    const int TE = tile_entries(a.m, a.overlap);
    const size_t smem = sizeof(float) * ((size_t)kRows * a.d_in + (size_t)kKC * 128 + (size_t)kRows * 128 +
                                         (size_t)TE * a.d_out);
    auto kern = compress_gated_kernel<Tin, OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.N_c + TE - 1) / TE), (unsigned)a.B);
    kern<<<grid, kThreads, smem, s>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_out(const GatedArgs& a, cudaStream_t s, const char** why) {
    switch (a.out_dt) {
        case DT_F32:
            if (std::is_same<Tin, float>::value) return launch_t<Tin, DT_F32>(a, s);
            break;
        case DT_BF16: return launch_t<Tin, DT_BF16>(a, s);
        case DT_E4M3: return launch_t<Tin, DT_E4M3>(a, s);
        case DT_E4M3H: return launch_t<Tin, DT_E4M3H>(a, s);
    }
    *why = "csa_compress_gated: unsupported (x_dt, out_dt) pair";
    return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_compress_gated(const GatedArgs& a, cudaStream_t s, const char** why) {
    if (a.N_c <= 0 || a.B <= 0) return cudaSuccess;
    if (a.x_dt == DT_F32) return launch_out<float>(a, s, why);
    if (a.x_dt == DT_BF16) return launch_out<__nv_bfloat16>(a, s, why);
    *why = "csa_compress_gated: x must be F32 or BF16";
    return cudaErrorNotSupported;
}

}  // namespace csa
