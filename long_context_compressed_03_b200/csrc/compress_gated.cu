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
// overlapping).  bf16 inputs: bf16 tensor-core MMAs (m16n8k16, fp32
// accumulation, the exact products of the bf16 values), x rows and the
// slice's weight columns staged in shared memory; fp32 inputs: a
// register-tiled fp32 product with 32-row chunks of the weights staged.  Each thread then folds its
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

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
                 "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared-memory bytes of one CTA.
template <typename Tin>
size_t gated_smem(int d_in, int d_out, int TE) {
    if (std::is_same<Tin, __nv_bfloat16>::value)    // xb [64][d_in+8], wb [128][d_in+8] (bf16)
        return 2 * ((size_t)64 * (d_in + 8) + (size_t)128 * (d_in + 8)) +
               4 * ((size_t)64 * 128 + (size_t)TE * d_out);
    return 4 * ((size_t)64 * d_in + (size_t)32 * 128 + (size_t)64 * 128 + (size_t)TE * d_out);
}

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
    constexpr bool kMma = std::is_same<Tin, __nv_bfloat16>::value;
    const int ld = d_in + 8;                         // bf16 row stride: conflict-free fragments
    // fp32 inputs: xs [kRows][d_in], ws [kKC][128]; bf16: xb [kRows][ld], wb [128][ld]
    float* xs = smem;
    float* ws = xs + kRows * d_in;
    __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(smem);
    __nv_bfloat16* wb = xb + kRows * ld;
    float* proj = kMma ? reinterpret_cast<float*>(wb + 128 * ld) : ws + kKC * 128;   // [kRows][128]
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
        if constexpr (kMma) {
            // the slice's weight columns, transposed to [column][k] (bf16)
            __syncthreads();                         // the previous slice's MMAs are done with wb
            for (int q = tid; q < d_in * ncols; q += kThreads) {
                const int k = q / ncols, j = q - k * ncols;
                const int grp = j / kDC, ec = j - grp * kDC;
                const bool gate = grp >= nh;
                const int half = gate ? grp - nh : grp;
                __nv_bfloat16 w = __float2bfloat16_rn(0.0f);
                if (ec < dc) w = (gate ? Wg : Wkv)[(size_t)k * cw + half * d_out + e0 + ec];
                wb[j * ld + k] = w;
            }
        }
        for (int r0 = p_lo; r0 < p_hi; r0 += kRows) {
            const int nr = min(kRows, p_hi - r0);
            __syncthreads();                         // xs / proj of the previous step consumed
          if constexpr (kMma) {
            // x rows (bf16, 16 bytes at a time), zero past the tile
            const int vpr = d_in / 8;                // 16-byte vectors per row
            for (int q = tid; q < kRows * vpr; q += kThreads) {
                const int r = q / vpr, v = q - r * vpr;
                uint4 val = make_uint4(0u, 0u, 0u, 0u);
                if (r < nr) val = *reinterpret_cast<const uint4*>(x + (size_t)(r0 + r) * d_in + 8 * v);
                *reinterpret_cast<uint4*>(xb + r * ld + 8 * v) = val;
            }
            __syncthreads();
            // warp w: rows 16 (w >> 1) .., columns 64 (w & 1) .. (8 tiles of 8)
            const int g = tx >> 2, tq = tx & 3;
            const int rt = ty >> 1, c0 = 64 * (ty & 1);
            if (c0 < ncols) {
                float acc[8][4];
#pragma unroll
                for (int t = 0; t < 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
                const __nv_bfloat16* ar = xb + (16 * rt + g) * ld + 2 * tq;
                for (int k0 = 0; k0 < d_in; k0 += 16) {
                    const uint32_t a0 = *reinterpret_cast<const uint32_t*>(ar + k0);
                    const uint32_t a1 = *reinterpret_cast<const uint32_t*>(ar + 8 * ld + k0);
                    const uint32_t a2 = *reinterpret_cast<const uint32_t*>(ar + k0 + 8);
                    const uint32_t a3 = *reinterpret_cast<const uint32_t*>(ar + 8 * ld + k0 + 8);
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        const __nv_bfloat16* br = wb + (c0 + 8 * t + g) * ld + k0 + 2 * tq;
                        mma_bf16(acc[t], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(br),
                                 *reinterpret_cast<const uint32_t*>(br + 8));
                    }
                }
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    float* pr = proj + (16 * rt + g) * 128 + c0 + 8 * t + 2 * tq;
                    *reinterpret_cast<float2*>(pr) = make_float2(acc[t][0], acc[t][1]);
                    *reinterpret_cast<float2*>(pr + 8 * 128) = make_float2(acc[t][2], acc[t][3]);
                }
            }
          } else {
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
    const size_t smem = gated_smem<Tin>(a.d_in, a.d_out, TE);
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
