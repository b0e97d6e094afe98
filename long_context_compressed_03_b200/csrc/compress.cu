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
#include "tc_common.cuh"

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

// ---------------------------------------------------------------- tensor-core path
// bf16 x and W: the projection runs on the tensor cores (mma.sync m16n8k16,
// bf16 operands, fp32 accumulate).  The pooled fp32 value is split into
// three bf16 parts, v = h1 + h2 + h3 exactly (8 + 8 + 8 significant bits;
// each residual is exact in fp32), and W is bf16 already, so the three
// products per term are exact and only the accumulation rounds -- fp32
// accuracy, as the FFMA path above.  A CTA owns E entries (E = 32 for small
// m; fewer for long blocks, so a CTA reads at most 64 KB of x); its x rows
// are summed with 16-byte loads, R rows per work item, all in flight.
constexpr int kME = 32;                  // entry rows of the MMA tile (two m16 tiles)

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
                 "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two fp32 values split into three bf16 pairs (lo element in the low half):
// v = h1 + h2 + h3 exactly for normal values.
__device__ __forceinline__ void split3(float v0, float v1, uint32_t& p1, uint32_t& p2, uint32_t& p3) {
    const __nv_bfloat16 a1 = __float2bfloat16_rn(v0), b1 = __float2bfloat16_rn(v1);
    const float r0 = v0 - __bfloat162float(a1), s0 = v1 - __bfloat162float(b1);
    const __nv_bfloat16 a2 = __float2bfloat16_rn(r0), b2 = __float2bfloat16_rn(s0);
    const __nv_bfloat16 a3 = __float2bfloat16_rn(r0 - __bfloat162float(a2));
    const __nv_bfloat16 b3 = __float2bfloat16_rn(s0 - __bfloat162float(b2));
    p1 = (uint32_t)__bfloat16_as_ushort(a1) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
    p2 = (uint32_t)__bfloat16_as_ushort(a2) | ((uint32_t)__bfloat16_as_ushort(b2) << 16);
    p3 = (uint32_t)__bfloat16_as_ushort(a3) | ((uint32_t)__bfloat16_as_ushort(b3) << 16);
}

// Shared memory of the tensor-core path: W (bf16, rows padded by 8), the
// partial block sums, the pooled rows (fp32, rows padded by 4); the output
// rows reuse the last two.
struct MmaSmem {
    int ws, ps;                      // row strides of W (bf16) and pooled (fp32), elements
    size_t w_bytes, sum_bytes, pool_bytes, bytes;
};
__host__ __device__ inline MmaSmem mma_smem(int d_in, int d_out, int G, int nb) {
    MmaSmem s;
    s.ws = d_out + 8;
    s.ps = d_in + 4;
    s.w_bytes = (size_t)d_in * s.ws * 2;
    s.sum_bytes = (size_t)G * nb * d_in * 4;
    s.pool_bytes = (size_t)kME * s.ps * 4;
    size_t tail = s.sum_bytes + s.pool_bytes;
    const size_t outs = (size_t)kME * d_out * 4;
    if (outs > tail) tail = outs;
    s.bytes = s.w_bytes + tail;
    return s;
}

template <int R, int OUT>
__global__ void __launch_bounds__(kThreads) compress_mma_kernel(CompressKArgs a, int E) {
    extern __shared__ __align__(16) uint8_t smem8[];
    const int d_in = a.d_in, d_out = a.d_out, m = a.m;
    const int G = m / R;                               // row groups of a block
    const int b = blockIdx.y;
    size_t tok0 = (size_t)b * a.n, ent0 = (size_t)b * a.N_c;
    int N_c = a.N_c;
    if (a.map.S) {
        tok0 = (size_t)a.map.tok[b];
        ent0 = (size_t)a.map.ent[b];
        N_c = (a.map.tok[b + 1] - a.map.tok[b]) / m;
    }
    const int i0 = blockIdx.x * E;
    if (i0 >= N_c) return;                             // a shorter packed sequence
    const int ne = min(E, N_c - i0);
    const int jb0 = a.overlap ? -1 : 0;                // block i0 - 1 when overlapping
    const int nb = ne - jb0;                           // blocks summed
    const MmaSmem L = mma_smem(d_in, d_out, G, nb);
    __nv_bfloat16* sW = reinterpret_cast<__nv_bfloat16*>(smem8);
    float* psum = reinterpret_cast<float*>(smem8 + L.w_bytes);            // [G][nb][d_in]
    float* pool = reinterpret_cast<float*>(smem8 + L.w_bytes + L.sum_bytes);  // [kME][ps]
    float* outs = reinterpret_cast<float*>(smem8 + L.w_bytes);            // [kME][d_out], later
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x) + tok0 * d_in;
    const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.W);
    const int tid = threadIdx.x;

    // ---- W, with 16-byte loads (L2-resident across CTAs), eight in flight per thread
    {
        const int c8s = d_out / 8, nw = d_in * c8s;
        for (int q0 = tid; q0 < nw; q0 += 8 * kThreads) {
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * kThreads;
                wv[i] = q < nw ? __ldg(reinterpret_cast<const uint4*>(W) + q) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * kThreads;
                if (q < nw) {
                    const int k = q / c8s, c8 = q - k * c8s;
                    *reinterpret_cast<uint4*>(sW + k * L.ws + c8 * 8) = wv[i];
                }
            }
        }
    }
    // ---- partial block sums: work item (group g, block jb, 16-byte piece f), R rows
    {
        const int pieces = d_in / 8;
        const int items = G * nb * pieces;
        constexpr int kPer = 16 / R;                   // items per thread with loads in flight together
        for (int w0 = tid; w0 < items; w0 += kThreads * kPer) {
            uint4 v[kPer][R];
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int w = w0 + q * kThreads;
                const int f = w % pieces, rest = w / pieces;
                const int jb = rest % nb, g = rest / nb;
                const int blk = i0 + jb0 + jb;
                const bool live = w < items && blk >= 0;
                const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)(live ? blk : 0) * m + g * R) * d_in) + f;
#pragma unroll
                for (int r = 0; r < R; ++r)
                    v[q][r] = live ? __ldg(src + (size_t)r * pieces) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int w = w0 + q * kThreads;
                if (w >= items) continue;
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
                for (int r = 0; r < R; ++r) Vec<__nv_bfloat16>::add(acc, v[q][r]);
                const int f = w % pieces, rest = w / pieces;
                float* dst = psum + (size_t)rest * d_in + f * 8;      // rest = g * nb + jb
                *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
        }
    }
    __syncthreads();
    // ---- pooled rows: (previous block + own block) / count; rows >= ne are 0
    for (int q = tid; q < kME * d_in; q += kThreads) {
        const int e = q / d_in, c = q - e * d_in;
        float v = 0.0f;
        if (e < ne) {
            float cur = 0.0f, prev = 0.0f;
            for (int g = 0; g < G; ++g) {
                cur += psum[((size_t)g * nb + e - jb0) * d_in + c];
                if (a.overlap) prev += psum[((size_t)g * nb + e - jb0 - 1) * d_in + c];
            }
            const int i = i0 + e;
            const int lo = a.overlap ? max(0, m * (i - 1)) : m * i;
            v = (a.overlap ? prev + cur : cur) / (float)(m * (i + 1) - lo);
        }
        pool[e * L.ps + c] = v;
    }
    __syncthreads();
    // ---- projection: warp w takes m16 tile (w % mtiles) and a range of n8 tiles
    const int warp = tid >> 5, lane = tid & 31;
    const int mtiles = ne > 16 ? 2 : 1;
    const int wpm = 8 / mtiles;                        // warps per m16 tile
    const int ncols = d_out / wpm;                     // a multiple of 8 (d_out % 64 == 0)
    const int mt = warp % mtiles, n0 = (warp / mtiles) * ncols;
    const int ntiles = ncols / 8;                      // 1 .. 8
    float acc[8][4];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
    const int g8 = lane >> 2, c2 = 2 * (lane & 3);
    const float* prow0 = pool + (mt * 16 + g8) * L.ps;
    const float* prow1 = prow0 + 8 * L.ps;
    const uint32_t sw_base = (uint32_t)__cvta_generic_to_shared(sW);
    for (int ks = 0; ks < d_in / 16; ++ks) {
        const int k0 = ks * 16 + c2;
        const float2 v00 = *reinterpret_cast<const float2*>(prow0 + k0);
        const float2 v10 = *reinterpret_cast<const float2*>(prow1 + k0);
        const float2 v01 = *reinterpret_cast<const float2*>(prow0 + k0 + 8);
        const float2 v11 = *reinterpret_cast<const float2*>(prow1 + k0 + 8);
        uint32_t A[3][4];
        split3(v00.x, v00.y, A[0][0], A[1][0], A[2][0]);
        split3(v10.x, v10.y, A[0][1], A[1][1], A[2][1]);
        split3(v01.x, v01.y, A[0][2], A[1][2], A[2][2]);
        split3(v11.x, v11.y, A[0][3], A[1][3], A[2][3]);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            if (2 * np >= ntiles) break;
            uint32_t b0, b1, b2, b3;
            const uint32_t addr = sw_base + (uint32_t)(((ks * 16 + (lane & 15)) * L.ws + n0 + np * 16 +
                                                        (lane >> 4) * 8) * 2);
            ldsm_x4_t(addr, b0, b1, b2, b3);
#pragma unroll
            for (int sp = 0; sp < 3; ++sp) {
                mma_bf16(acc[2 * np], A[sp], b0, b1);
                if (2 * np + 1 < ntiles) mma_bf16(acc[2 * np + 1], A[sp], b2, b3);
            }
        }
    }
    __syncthreads();                                   // pooled rows and sums are no longer read
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        if (t >= ntiles) break;
        const int col = n0 + t * 8 + c2;
        const int r0 = mt * 16 + g8, r1 = r0 + 8;
        if (r0 < ne) *reinterpret_cast<float2*>(outs + r0 * d_out + col) = make_float2(acc[t][0], acc[t][1]);
        if (r1 < ne) *reinterpret_cast<float2*>(outs + r1 * d_out + col) = make_float2(acc[t][2], acc[t][3]);
    }
    __syncthreads();
    store_entry_rows<OUT, kThreads>(outs, ne, d_out, a.out, a.out_row_scale, ent0 + i0, a.hnorm);
}

// ---------------------------------------------------------------- streaming path
// The same arithmetic as compress_mma_kernel, persistent: one CTA per SM
// walks the tiles t = blockIdx.x, + gridDim.x, ... of every batch element.
// W is staged once per CTA.  A tile's rows of x are one contiguous range of
// global memory, so one thread brings them into shared memory with a single
// bulk copy (TMA, no multicast) on an mbarrier; the next tile's copy is in
// flight while a tile is summed, projected and stored (two slab buffers).
// The pooled rows are split into their three bf16 planes once, in shared
// memory, and read by ldmatrix.
struct StreamArgs {
    CompressKArgs a;
    int E;                  // entries per tile
    int tiles_per_seq;
    int tiles;              // B * tiles_per_seq
    uint32_t* err;
    uint64_t wait_ns;
};

struct StreamSmem {
    int ws, as;
    size_t w_bytes, slab_bytes, sum_bytes, plane_bytes, bar_off, bytes;
};
__host__ __device__ inline StreamSmem stream_smem(int d_in, int d_out, int m, int G, int E) {
    StreamSmem s;
    s.ws = d_out + 8;
    s.as = d_in + 8;
    s.w_bytes = (size_t)d_in * s.ws * 2;
    s.slab_bytes = (size_t)(E + 1) * m * d_in * 2;
    s.sum_bytes = (size_t)G * (E + 1) * d_in * 4;
    s.plane_bytes = (size_t)3 * kME * s.as * 2;
    size_t tail = s.sum_bytes + s.plane_bytes;
    const size_t outs = (size_t)kME * d_out * 4;
    if (outs > tail) tail = outs;
    s.bar_off = s.w_bytes + 2 * s.slab_bytes + tail;
    s.bytes = s.bar_off + 32 + kME * 4;      // barriers, abort flag, 1 / count per entry
    return s;
}

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <int R, int OUT>
__global__ void __launch_bounds__(kThreads, 1) compress_stream_kernel(StreamArgs sa) {
    extern __shared__ __align__(16) uint8_t smem8[];
    const CompressKArgs& a = sa.a;
    const int d_in = a.d_in, d_out = a.d_out, m = a.m, E = sa.E;
    const int G = m / R;
    const int jb0 = a.overlap ? -1 : 0;
    const StreamSmem L = stream_smem(d_in, d_out, m, G, E);
    __nv_bfloat16* sW = reinterpret_cast<__nv_bfloat16*>(smem8);
    uint8_t* slab0 = smem8 + L.w_bytes;                                     // [2][(E+1) m][d_in] bf16
    float* psum = reinterpret_cast<float*>(smem8 + L.w_bytes + 2 * L.slab_bytes);   // [G][E+1][d_in]
    __nv_bfloat16* planes = reinterpret_cast<__nv_bfloat16*>(
        smem8 + L.w_bytes + 2 * L.slab_bytes + L.sum_bytes);                // [3][kME][as]
    float* outs = psum;                                                     // [kME][d_out], later
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem8 + L.bar_off);         // [2]
    volatile int* abort = reinterpret_cast<volatile int*>(smem8 + L.bar_off + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(a.x);
    const size_t row_bytes = (size_t)d_in * 2;

    // a tile's rows: blocks i0 + jb0 .. i0 + ne - 1 of element b (block -1 absent)
    auto tile_of = [&](int t, int& b, int& i0, int& ne) {
        b = t / sa.tiles_per_seq;
        i0 = (t - b * sa.tiles_per_seq) * E;
        ne = min(E, a.N_c - i0);
    };
    auto issue = [&](int t, int buf) {           // one thread
        int b, i0, ne;
        tile_of(t, b, i0, ne);
        const int blk0 = max(i0 + jb0, 0);
        const int nblk = i0 + ne - blk0;
        const uint32_t bytes = (uint32_t)((size_t)nblk * m * row_bytes);
        uint8_t* dst = slab0 + (size_t)buf * L.slab_bytes + (size_t)(blk0 - (i0 + jb0)) * m * row_bytes;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(xg + ((size_t)b * a.n + (size_t)blk0 * m) * d_in);
        tc::mbar_arrive_expect_tx(&bar[buf], bytes);
        bulk_copy(dst, src, bytes, &bar[buf]);
    };

    if (tid == 0) {
        tc::mbar_init(&bar[0], 1);
        tc::mbar_init(&bar[1], 1);
        *abort = (*reinterpret_cast<volatile uint32_t*>(sa.err) != 0u) ? 1 : 0;
        tc::fence_barrier_init();
    }
    __syncthreads();
    int issued = 0;                                   // copies issued (thread 0)
    if (tid == 0 && blockIdx.x < sa.tiles && !*abort) { issue(blockIdx.x, 0); issued = 1; }
    // ---- W once, eight 16-byte loads in flight per thread
    {
        const int c8s = d_out / 8, nw = d_in * c8s;
        const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.W);
        for (int q0 = tid; q0 < nw; q0 += 8 * kThreads) {
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * kThreads;
                wv[i] = q < nw ? __ldg(reinterpret_cast<const uint4*>(W) + q) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * kThreads;
                if (q < nw) {
                    const int k = q / c8s, c8 = q - k * c8s;
                    *reinterpret_cast<uint4*>(sW + k * L.ws + c8 * 8) = wv[i];
                }
            }
        }
    }
    // per-thread coordinates of the sums and the pooled rows (one division each)
    const int pieces = d_in / 8;
    const int sum_f = tid % pieces, sum_q0 = tid / pieces, sum_step = kThreads / pieces;
    const int dh = d_in / 2;
    const int pool_c = 2 * (tid % dh), pool_e0 = tid / dh, pool_estep = kThreads / dh;
    float* inv_cnt = reinterpret_cast<float*>(smem8 + L.bar_off + 32);   // [kME]
    int k = 0;
    for (int t = blockIdx.x; t < sa.tiles; t += gridDim.x, ++k) {
        const int buf = k & 1;
        // the next tile's rows into the other buffer (its last reader finished
        // at the end of the previous tile)
        if (tid == 0 && t + (int)gridDim.x < sa.tiles && !*abort) { issue(t + gridDim.x, buf ^ 1); ++issued; }
        // this tile's rows have landed (every thread waits: bounded)
        const bool okw = tc::mbar_wait(&bar[buf], (k >> 1) & 1, abort, sa.err, sa.wait_ns);
        if (__syncthreads_or(!okw)) break;
        int b, i0, ne;
        tile_of(t, b, i0, ne);
        const int nb = ne - jb0;
        const __nv_bfloat16* slab = reinterpret_cast<const __nv_bfloat16*>(slab0 + (size_t)buf * L.slab_bytes);
        // ---- partial block sums from shared memory: item (g, jb, 16-byte piece f), R rows;
        //      a thread keeps its piece and steps (g, jb) without divisions
        {
            const int items = G * nb;
            int q = sum_q0, jb = sum_q0, g = 0;
            while (jb >= nb) { jb -= nb; ++g; }
            for (; q < items; q += sum_step) {
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
                if (i0 + jb0 + jb >= 0) {
                    const uint4* src = reinterpret_cast<const uint4*>(slab + ((size_t)jb * m + g * R) * d_in) + sum_f;
#pragma unroll
                    for (int r = 0; r < R; ++r) Vec<__nv_bfloat16>::add(acc, src[(size_t)r * pieces]);
                }
                float* dst = psum + (size_t)(g * nb + jb) * d_in + sum_f * 8;
                *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
                jb += sum_step;
                while (jb >= nb) { jb -= nb; ++g; }
            }
        }
        // the tile's 1 / count per entry (exact for the power-of-two counts of
        // m = 2^j; otherwise one more rounding, inside the same error bound)
        if (tid < kME) {
            const int i = i0 + tid;
            const int lo = a.overlap ? max(0, m * (i - 1)) : m * i;
            inv_cnt[tid] = 1.0f / (float)(m * (i + 1) - lo);
        }
        __syncthreads();
        // ---- pooled rows split into three bf16 planes (rows >= ne are 0); a
        //      thread keeps its column pair and steps the entry
        for (int e = pool_e0; e < kME; e += pool_estep) {
            float v0 = 0.0f, v1 = 0.0f;
            if (e < ne) {
                float c0 = 0.0f, c1 = 0.0f, p0 = 0.0f, p1 = 0.0f;
                for (int g = 0; g < G; ++g) {
                    const float2 cur = *reinterpret_cast<const float2*>(psum + ((size_t)g * nb + e - jb0) * d_in + pool_c);
                    c0 += cur.x;
                    c1 += cur.y;
                    if (a.overlap) {
                        const float2 pr = *reinterpret_cast<const float2*>(psum + ((size_t)g * nb + e - jb0 - 1) * d_in + pool_c);
                        p0 += pr.x;
                        p1 += pr.y;
                    }
                }
                const float ic = inv_cnt[e];
                v0 = (a.overlap ? p0 + c0 : c0) * ic;
                v1 = (a.overlap ? p1 + c1 : c1) * ic;
            }
            uint32_t h1, h2, h3;
            split3(v0, v1, h1, h2, h3);
            const size_t o = (size_t)e * L.as + pool_c;
            *reinterpret_cast<uint32_t*>(planes + o) = h1;
            *reinterpret_cast<uint32_t*>(planes + (size_t)kME * L.as + o) = h2;
            *reinterpret_cast<uint32_t*>(planes + 2 * (size_t)kME * L.as + o) = h3;
        }
        __syncthreads();
        // ---- projection: warp w takes m16 tile (w % mtiles) and a range of n8 tiles
        const int mtiles = ne > 16 ? 2 : 1;
        const int wpm = 8 / mtiles;
        const int ncols = d_out / wpm;
        const int mt = warp % mtiles, n0 = (warp / mtiles) * ncols;
        const int ntiles = ncols / 8;
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
        const uint32_t sw_base = tc::smem_u32(sW);
        const uint32_t pl_base = tc::smem_u32(planes);
        for (int ks = 0; ks < d_in / 16; ++ks) {
            uint32_t A[3][4];
#pragma unroll
            for (int sp = 0; sp < 3; ++sp) {
                const uint32_t addr = pl_base + (uint32_t)((((size_t)sp * kME + mt * 16 + (lane & 15)) * L.as +
                                                           ks * 16 + (lane >> 4) * 8) * 2);
                ldsm_x4(addr, A[sp][0], A[sp][1], A[sp][2], A[sp][3]);
            }
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                if (2 * np >= ntiles) break;
                uint32_t b0, b1, b2, b3;
                const uint32_t addr = sw_base + (uint32_t)(((ks * 16 + (lane & 15)) * L.ws + n0 + np * 16 +
                                                            (lane >> 4) * 8) * 2);
                ldsm_x4_t(addr, b0, b1, b2, b3);
#pragma unroll
                for (int sp = 0; sp < 3; ++sp) {
                    mma_bf16(acc[2 * np], A[sp], b0, b1);
                    if (2 * np + 1 < ntiles) mma_bf16(acc[2 * np + 1], A[sp], b2, b3);
                }
            }
        }
        __syncthreads();                               // sums and planes are no longer read
        {
            const int g8 = lane >> 2, c2 = 2 * (lane & 3);
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) {
                if (tt >= ntiles) break;
                const int col = n0 + tt * 8 + c2;
                const int r0 = mt * 16 + g8, r1 = r0 + 8;
                if (r0 < ne) *reinterpret_cast<float2*>(outs + r0 * d_out + col) = make_float2(acc[tt][0], acc[tt][1]);
                if (r1 < ne) *reinterpret_cast<float2*>(outs + r1 * d_out + col) = make_float2(acc[tt][2], acc[tt][3]);
            }
        }
        __syncthreads();
        store_entry_rows<OUT, kThreads>(outs, ne, d_out, a.out, a.out_row_scale,
                                        (size_t)b * a.N_c + i0, a.hnorm);
        __syncthreads();                               // outs (and this slab) free for the next tile
    }
    // copies still in flight (an abort) land before the CTA's shared memory is given up
    if (tid == 0) {
        volatile int never = 0;
        for (int j = max(0, issued - 2); j < issued; ++j)
            tc::mbar_wait(&bar[j & 1], (j >> 1) & 1, &never, sa.err);
    }
    __syncthreads();
}

template <int R, int OUT>
cudaError_t launch_stream_r(const CompressKArgs& a, cudaStream_t s) {
    int E = (int)(65536 / ((size_t)a.m * a.d_in * 2));
    E = E < 1 ? 1 : (E > kME ? kME : E);
    const int G = a.m / R;
    const StreamSmem L = stream_smem(a.d_in, a.d_out, a.m, G, E);
    uint32_t* err = device_error_word();
    if (!err) return cudaErrorUnknown;
    StreamArgs sa;
    sa.a = a;
    sa.E = E;
    sa.tiles_per_seq = (a.N_c + E - 1) / E;
    sa.tiles = a.B * sa.tiles_per_seq;
    sa.err = err;
    sa.wait_ns = wait_limit_ns();
    auto kern = compress_stream_kernel<R, OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.bytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = sa.tiles < sms ? sa.tiles : sms;
    kern<<<grid, kThreads, L.bytes, s>>>(sa);
    count_launch();
    return cudaGetLastError();
}

template <int OUT>
cudaError_t launch_stream(const CompressKArgs& a, cudaStream_t s) {
    const int m = a.m;
    if (m % 16 == 0) return launch_stream_r<16, OUT>(a, s);
    if (m % 8 == 0) return launch_stream_r<8, OUT>(a, s);
    if (m % 4 == 0) return launch_stream_r<4, OUT>(a, s);
    if (m % 2 == 0) return launch_stream_r<2, OUT>(a, s);
    return launch_stream_r<1, OUT>(a, s);
}

// The streaming path: unpacked calls whose tiles fit the shared memory (two
// row slabs, W, sums and planes) and whose rows are 16-byte multiples.
bool stream_path(const CompressArgs& a) {
    if (a.vl || a.B <= 0 || a.N_c <= 0) return false;
    int E = (int)(65536 / ((size_t)a.m * a.d_in * 2));
    E = E < 1 ? 1 : (E > kME ? kME : E);
    int R = 16;
    while (a.m % R) R >>= 1;
    const StreamSmem L = stream_smem(a.d_in, a.d_out, a.m, a.m / R, E);
    return L.bytes <= 227 * 1024;
}

template <int R, int OUT>
cudaError_t launch_mma_r(const CompressKArgs& a, cudaStream_t s) {
    // entries per CTA: at most 64 KB of x (and 32, the MMA tile)
    int E = (int)(65536 / ((size_t)a.m * a.d_in * 2));
    E = E < 1 ? 1 : (E > kME ? kME : E);
    const int G = a.m / R;
    const MmaSmem L = mma_smem(a.d_in, a.d_out, G, E + (a.overlap ? 1 : 0));
    auto kern = compress_mma_kernel<R, OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((a.N_c + E - 1) / E, a.B);
    kern<<<grid, kThreads, L.bytes, s>>>(a, E);
    count_launch();
    return cudaGetLastError();
}

template <int OUT>
cudaError_t launch_mma(const CompressKArgs& a, cudaStream_t s) {
    const int m = a.m;
    if (m % 16 == 0) return launch_mma_r<16, OUT>(a, s);
    if (m % 8 == 0) return launch_mma_r<8, OUT>(a, s);
    if (m % 4 == 0) return launch_mma_r<4, OUT>(a, s);
    if (m % 2 == 0) return launch_mma_r<2, OUT>(a, s);
    return launch_mma_r<1, OUT>(a, s);
}

// The tensor-core path serves bf16 x / W with d_in a multiple of 16 and d_out
// a multiple of 64, both at most 256 (shared memory: W, sums, pooled rows).
bool mma_path(const CompressArgs& a) {
    return a.x_dt == DT_BF16 && a.d_in % 16 == 0 && a.d_out % 64 == 0 && a.d_in <= 256 &&
           a.d_out <= 256;
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
    } else if (a.x_dt == DT_BF16 && mma_path(a)) {
        CompressKArgs k;
        static_cast<CompressArgs&>(k) = a;
        if (a.vl) k.map = *a.vl;
        if (stream_path(a)) {
            if (a.out_dt == DT_BF16) return launch_stream<DT_BF16>(k, s);
            if (a.out_dt == DT_E4M3) return launch_stream<DT_E4M3>(k, s);
            if (a.out_dt == DT_E4M3H) return launch_stream<DT_E4M3H>(k, s);
        }
        if (a.out_dt == DT_BF16) return launch_mma<DT_BF16>(k, s);
        if (a.out_dt == DT_E4M3) return launch_mma<DT_E4M3>(k, s);
        if (a.out_dt == DT_E4M3H) return launch_mma<DT_E4M3H>(k, s);
    } else if (a.x_dt == DT_BF16) {
        if (a.out_dt == DT_BF16) return launch_t<__nv_bfloat16, DT_BF16>(a, s);
        if (a.out_dt == DT_E4M3) return launch_t<__nv_bfloat16, DT_E4M3>(a, s);
        if (a.out_dt == DT_E4M3H) return launch_t<__nv_bfloat16, DT_E4M3H>(a, s);
    }
    *why = "csa_compress: unsupported (x_dt, out_dt) pair";
    return cudaErrorNotSupported;
}

}  // namespace csa
