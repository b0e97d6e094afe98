// compress.cu -- stage 1: overlapping mean-pool compression + projection.
//
// out[b, i, :] = (mean_{p in win(i)} x[b, p, :]) @ W
//   overlap: win(i) = [m(i-1), m(i+1)) ∩ [0, n)  -- own block + previous block
//   plain:   win(i) = [m i, m(i+1))
// ("百万上下文从「奢侈品」变「日用品」…" §3.2 mean pool + projection;
//  "DS-V4 分析&学习" §1.3 2m-position overlap; "DeepSeek V4 CSA + CP 迁移到 HP…"
//  §3.2 ratio 4 overlapping, ratio 128 not.)
//
// One CTA owns a tile of 32 consecutive entries of one batch element.
//  * Block sums: the tile's blocks (and, when overlapping, the block before
//    it) are summed over their m rows in fp32, each thread taking 16-byte
//    pieces (8 bf16 / 4 fp32 features) of several blocks with all their loads
//    in flight, so x is read once in wide coalesced loads; an entry's pooled
//    row is then (previous block + own block) / count.
//  * Projection: a register-tiled fp32 product with W staged in shared memory
//    32 rows at a time; each thread accumulates 4 entries x 4 outputs, the
//    pooled values of a warp's entries being broadcast reads.
//  * Epilogue: bf16/fp32 stores, or per-row amax across a warp and E4M3
//    quantisation (IEEE division, round to nearest even, saturating), for the
//    Hadamard type after the warp rotates the row in shared memory.
#include "common.cuh"
#include "entry_epilogue.cuh"
#include "kernels.h"

namespace csa {
namespace {

// The kernel's arguments: the call's, plus the packed-sequence map by value.
struct CompressKArgs : CompressArgs {
    VarlenMap map;
};

constexpr int kThreads = 256;
constexpr int kTile = 32;   // entries per CTA
constexpr int kKC = 32;     // rows of W staged per step

// 16 bytes of x as fp32 features: 8 bf16 or 4 fp32.
template <typename Tin> struct Vec;
template <> struct Vec<__nv_bfloat16> {
    static constexpr int kN = 8;
    __device__ static void add(float* acc, uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(w[i] << 16);
            acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <> struct Vec<float> {
    static constexpr int kN = 4;
    __device__ static void add(float* acc, uint4 v) {
        acc[0] += __uint_as_float(v.x);
        acc[1] += __uint_as_float(v.y);
        acc[2] += __uint_as_float(v.z);
        acc[3] += __uint_as_float(v.w);
    }
};

template <typename Tin, int OUT>
__global__ void __launch_bounds__(kThreads) compress_kernel(CompressKArgs a) {
    extern __shared__ float smem[];
    constexpr int VN = Vec<Tin>::kN;
    const int d_in = a.d_in, d_out = a.d_out, m = a.m;
    const int b = blockIdx.y;
    // element b (or packed sequence b): its tokens start at tok0, its entries at ent0
    size_t tok0 = (size_t)b * a.n, ent0 = (size_t)b * a.N_c;
    int N_c = a.N_c;
    if (a.map.S) {
        tok0 = (size_t)a.map.tok[b];
        ent0 = (size_t)a.map.ent[b];
        N_c = (a.map.tok[b + 1] - a.map.tok[b]) / m;
    }
    const int i0 = blockIdx.x * kTile;
    if (i0 >= N_c) return;                         // a shorter packed sequence
    const int ne = min(kTile, N_c - i0);
    float* bsum = smem;                            // [kTile + 1][d_in]: block sums (block i0 - 1 first)
    float* pooled = bsum + (kTile + 1) * d_in;     // [kTile][d_in]
    float* wst = pooled + kTile * d_in;            // [kKC][128]
    float* outs = wst + kKC * 128;                 // [kTile][d_out]
    const Tin* x = static_cast<const Tin*>(a.x) + tok0 * d_in;
    const Tin* W = static_cast<const Tin*>(a.W);
    const int tid = threadIdx.x;

    // ---- block sums: work item (block jb of the tile, 16-byte piece f)
    {
        const int pieces = d_in / VN;                    // 16-byte pieces of a row
        const int jb0 = a.overlap ? -1 : 0;              // block i0 - 1 when overlapping
        const int nb = ne - jb0;                         // blocks to sum
        const int items = nb * pieces;
        constexpr int kPer = 4;                          // items per thread with loads in flight together
        for (int w0 = tid; w0 < items; w0 += kThreads * kPer) {
            float acc[kPer][VN];
            int jbs[kPer], fs[kPer];
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int w = w0 + q * kThreads;
                jbs[q] = w < items ? w / pieces + jb0 : -2;
                fs[q] = w < items ? w % pieces : 0;
#pragma unroll
                for (int v = 0; v < VN; ++v) acc[q][v] = 0.0f;
            }
            for (int r = 0; r < m; ++r) {
                uint4 vals[kPer];
#pragma unroll
                for (int q = 0; q < kPer; ++q) {
                    const int blk = i0 + jbs[q];             // the block's index in the sequence
                    vals[q] = (jbs[q] >= jb0 && blk >= 0)
                        ? __ldg(reinterpret_cast<const uint4*>(x + ((size_t)blk * m + r) * d_in) + fs[q])
                        : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int q = 0; q < kPer; ++q) Vec<Tin>::add(acc[q], vals[q]);
            }
#pragma unroll
            for (int q = 0; q < kPer; ++q)
                if (jbs[q] >= jb0) {
#pragma unroll
                    for (int v = 0; v < VN; ++v) bsum[(jbs[q] - jb0) * d_in + fs[q] * VN + v] = acc[q][v];
                }
        }
        __syncthreads();
        // pooled rows: (previous block + own block) / count (own block alone when not overlapping)
        for (int q = tid; q < ne * d_in; q += kThreads) {
            const int e = q / d_in, c = q - e * d_in;
            const int i = i0 + e;
            const float cur = bsum[(e - jb0) * d_in + c];
            const int lo = a.overlap ? max(0, m * (i - 1)) : m * i;
            const float cnt = (float)(m * (i + 1) - lo);
            pooled[q] = (a.overlap ? bsum[(e - jb0 - 1) * d_in + c] + cur : cur) / cnt;
        }
    }
    // ---- projection: outs[e][o] = sum_k pooled[e][k] W[k][o]
    const int ty = tid >> 5, tx = tid & 31;            // entries 4 ty .. +3, outputs ob + 4 tx .. +3
    for (int ob = 0; ob < d_out; ob += 128) {
        const int ow = min(128, d_out - ob);
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.0f;
        for (int k0 = 0; k0 < d_in; k0 += kKC) {
            const int kc = min(kKC, d_in - k0);        // 16 or 32 (d_in is a multiple of 16)
            __syncthreads();                           // pooled ready / previous W chunk consumed
            for (int q = tid; q < kc * ow; q += kThreads) {
                const int kr = q / ow, oc = q - kr * ow;
                wst[kr * 128 + oc] = to_f32(W[(size_t)(k0 + kr) * d_out + ob + oc]);
            }
            __syncthreads();
            if (4 * tx < ow) {
#pragma unroll 8
                for (int kk = 0; kk < kc; ++kk) {
                    const float4 w4 = *reinterpret_cast<const float4*>(wst + kk * 128 + 4 * tx);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float pv = pooled[(4 * ty + r) * d_in + k0 + kk];
                        acc[r][0] = fmaf(pv, w4.x, acc[r][0]);
                        acc[r][1] = fmaf(pv, w4.y, acc[r][1]);
                        acc[r][2] = fmaf(pv, w4.z, acc[r][2]);
                        acc[r][3] = fmaf(pv, w4.w, acc[r][3]);
                    }
                }
            }
        }
        if (4 * tx < ow) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
                *reinterpret_cast<float4*>(outs + (4 * ty + r) * d_out + ob + 4 * tx) =
                    make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        }
    }
    __syncthreads();

    store_entry_rows<OUT, kThreads>(outs, ne, d_out, a.out, a.out_row_scale, ent0 + i0, a.hnorm);
}

template <typename Tin, int OUT>
cudaError_t launch_t(const CompressArgs& args, cudaStream_t s) {
    CompressKArgs a;
    static_cast<CompressArgs&>(a) = args;
    if (args.vl) a.map = *args.vl;
    const size_t smem = sizeof(float) * ((size_t)(2 * kTile + 1) * a.d_in + (size_t)kKC * 128 +
                                         (size_t)kTile * a.d_out);
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
        if (a.out_dt == DT_E4M3H) return launch_t<float, DT_E4M3H>(a, s);
    } else if (a.x_dt == DT_BF16) {
        if (a.out_dt == DT_BF16) return launch_t<__nv_bfloat16, DT_BF16>(a, s);
        if (a.out_dt == DT_E4M3) return launch_t<__nv_bfloat16, DT_E4M3>(a, s);
        if (a.out_dt == DT_E4M3H) return launch_t<__nv_bfloat16, DT_E4M3H>(a, s);
    }
    *why = "csa_compress: unsupported (x_dt, out_dt) pair";
    return cudaErrorNotSupported;
}

}  // namespace csa
