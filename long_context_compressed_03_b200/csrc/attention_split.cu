// attention_split.cu -- stage 3 for few query rows (decode): the keys of one
// query row are split over the CTAs of a thread-block cluster, each CTA runs
// the joint softmax over its share on the tensor cores, and the partial
// softmax states are merged through distributed shared memory.
//
// For query row (b, q) at position t and head h (one shared K = V head):
//   o[h] = sum_s softmax_s(scale * q[h] . key_s) key_s
// over the multiset {selected or visible compressed entries} ∪ {window rows}
// ("DS-V4 分析&学习" §1.2 joint softmax over compressed + window keys, §1.4
//  HCA over every visible entry; "百万上下文从「奢侈品」变「日用品」…" §4.3 window
//  [max(0, t-W+1), t], §5.2 1/sqrt(head_dim)).
//
// Decode has one query per sequence, so a CTA per row would leave most SMs
// idle while each streams hundreds of KB of keys.  Here row r's virtual key
// list (compressed part, then window part) is cut into C contiguous chunks,
// one per CTA of a C-CTA cluster.  Each CTA:
//   * stages its chunk's row codes (entry, raw row or invalid) in shared memory,
//   * streams 64-key tiles through a 3-stage cp.async ring (rows gathered by
//     index for CSA, contiguous for HCA and the window), XOR-swizzled so the
//     ldmatrix reads are conflict-free,
//   * computes S = Q K^T and O += P V with bf16 mma.sync (one warp per 16
//     heads, fp32 accumulators in registers) under an online base-2 softmax,
//   * publishes (running max m, sum of rounded weights l_r, exact sum l_e,
//     unnormalised O) in its shared memory.
// After a cluster barrier CTA c merges heads [c H/C, (c+1) H/C) from all C
// partial states (read over DSMEM) and writes o and the log-sum-exp.  O is
// normalised by l_r, the sum of the bf16-rounded weights the PV products
// used, so the output is an exact convex combination of the keys; the LSE
// uses the exact sum l_e.
//
// Decode is bound by HBM (about 128 flop per byte of keys); at one 64-head
// query per sequence the per-CTA tiles are too small for 128-row tcgen05
// tiles, and warp-level MMA keeps the tensor work well under the stream time.
#include <cooperative_groups.h>
#include <math.h>

#include <algorithm>

#include "attn_rows.cuh"
#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa {
namespace {

constexpr int kBN = 64;           // keys per tile
constexpr int kStages = 3;
constexpr int kMaxChunk = 4096;   // keys per CTA (row codes staged in shared memory)
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory plan (bytes): key ring, then row codes and validity words.
template <int D>
struct Plan {
    static constexpr int kTileBytes = kBN * D * 2;
    static constexpr int kRingBytes = kStages * kTileBytes;
    static constexpr int kOStride = D + 8;   // fp32 partial-O row stride (floats)
    static_assert(64 * kOStride * 4 <= kRingBytes || D == 64, "partial O must fit the key ring");
};

// Resident CTAs per SM the register budget is sized for (64 heads: 128 threads).
template <int H>
constexpr int min_blocks() { return H <= 64 ? 3 : 1; }

struct RowState {          // per-head partial softmax state of this CTA
    float m, lr, le;
};

template <int H, int D>
__global__ void __launch_bounds__(H * 2, min_blocks<H>()) attn_split_kernel(AttnArgs a, int max_chunk) {
    constexpr int kThreads = H * 2;
    constexpr int kKS = D / 16;     // k-steps of QK^T
    constexpr int kND = D / 8;      // n-blocks of O
    constexpr int kChunks = D / 8;  // 16-byte pieces per key row
    constexpr int kOS = D + 8;
    using P = Plan<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* ring = smem;
    float* sO = reinterpret_cast<float*>(smem);                            // reuses the ring
    uint8_t* sQ = smem + P::kRingBytes;                                    // [H][D] bf16, swizzled
    RowState* sSt = reinterpret_cast<RowState*>(sQ + H * D * 2);           // [H]
    int* sRow = reinterpret_cast<int*>(sSt + H);                           // [max_chunk]
    uint32_t* sValid = reinterpret_cast<uint32_t*>(sRow + max_chunk);      // [max_chunk / 32]

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int b = row / a.n_q;
    const int t = a.q_pos ? a.q_pos[row] : a.pos0 + (row - b * a.n_q);
    const RowKeys rk = row_keys(a, b, t);
    const int T = rk.n_comp + rk.n_win;
    const int ch = ((T + C - 1) / C + kBN - 1) / kBN * kBN;
    const int lo = min(T, rank * ch), hi = min(T, lo + ch);
    const int ntile = (hi - lo + kBN - 1) / kBN;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tq = lane & 3;

    using T16 = __nv_bfloat16;
    const T16* kvc = static_cast<const T16*>(a.kv_c);         // rows from cache_row()
    const T16* kvr = static_cast<const T16*>(a.kv_raw) + (size_t)b * a.L_raw * D;

    // ---- row codes: >= 0 physical row of a compressed entry, <= -2 raw row
    //      -(code + 2), -1 none
    for (int i0 = 0; i0 < ntile * kBN; i0 += kThreads) {
        const int i = i0 + tid;
        const int kk = lo + i;
        int code = -1;
        if (i < ntile * kBN && kk < hi) {
            if (kk < rk.n_comp) {
                const int s = a.dense ? kk : a.idx[(size_t)row * a.topk + kk];
                code = (s >= 0 && s < a.N_cap) ? (int)cache_row(a.pages, a.N_cap, b, s) : -1;
            } else {
                code = -(rk.win_lo + kk - rk.n_comp) - 2;
            }
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, code != -1);
        if (i < ntile * kBN) {
            sRow[i] = code;
            if (lane == 0) sValid[i >> 5] = bal;
        }
    }
    __syncthreads();

    auto load_tile = [&](int j, int st) {
        uint8_t* dst0 = ring + st * P::kTileBytes;
#pragma unroll 4
        for (int c = tid; c < kBN * kChunks; c += kThreads) {
            const int key = c / kChunks, piece = c - key * kChunks;
            const int code = sRow[j * kBN + key];
            uint8_t* dst = dst0 + key * D * 2 + ((piece ^ (key & 7)) << 4);
            const T16* src = code >= 0 ? kvc + (size_t)code * D : (code <= -2 ? kvr + (size_t)(-code - 2) * D : nullptr);
            if (src)
                cp_async16(smem_u32(dst), src + piece * 8);
            else
                *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
    };

    // ---- Q rows of all heads into shared memory (same swizzle as the key tiles)
    {
        const T16* q = static_cast<const T16*>(a.q) + (size_t)row * H * D;
        for (int c = tid; c < H * kChunks; c += kThreads) {
            const int h = c / kChunks, piece = c - h * kChunks;
            cp_async16(smem_u32(sQ + h * D * 2 + ((piece ^ (h & 7)) << 4)), q + (size_t)h * D + piece * 8);
        }
    }
    const int h0 = warp * 16;
    const uint32_t qbase = smem_u32(sQ);

    float o[kND][4];
#pragma unroll
    for (int i = 0; i < kND; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY;       // rows g, g + 8 (base-2 domain)
    float lr0 = 0.f, lr1 = 0.f, le0 = 0.f, le1 = 0.f;
    const float sl2 = a.scale * kLog2e;

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < ntile) load_tile(s, s);
        cp_async_commit();
    }

    for (int j = 0; j < ntile; ++j) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        if (j + kStages - 1 < ntile) load_tile(j + kStages - 1, (j + kStages - 1) % kStages);
        cp_async_commit();

        const uint32_t kbase = smem_u32(ring + (j % kStages) * P::kTileBytes);
        // ---- S = Q K^T : 16 heads x 64 keys
        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.0f;
        {
            const int mi = lane >> 3, rr = lane & 7;
            const int qh = h0 + rr + (mi & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < kKS; ++ks) {
                // A fragment of the warp's 16 heads: (h, k lo), (h+8, k lo), (h, k hi), (h+8, k hi)
                uint32_t qa[4];
                const int qp = ks * 2 + (mi >> 1);
                ldsm_x4(qbase + qh * D * 2 + ((qp ^ (qh & 7)) << 4), qa[0], qa[1], qa[2], qa[3]);
#pragma unroll
                for (int nbp = 0; nbp < 4; ++nbp) {
                    const int key = nbp * 16 + rr + (mi >> 1) * 8;
                    const int piece = ks * 2 + (mi & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + key * D * 2 + ((piece ^ (key & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(s[2 * nbp], qa, b0, b1);
                    mma_bf16(s[2 * nbp + 1], qa, b2, b3);
                }
            }
        }
        // ---- mask (only tiles with invalid slots), online softmax (rows g, g + 8)
        const uint32_t v_lo = sValid[j * 2], v_hi = sValid[j * 2 + 1];
        if ((v_lo & v_hi) != 0xffffffffu) {
#pragma unroll
            for (int nb = 0; nb < 8; ++nb) {
                const uint32_t word = nb < 4 ? v_lo : v_hi;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int bit = (nb & 3) * 8 + 2 * tq + (e & 1);
                    if (!((word >> bit) & 1u)) s[nb][e] = -INFINITY;
                }
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nb = 0; nb < 8; ++nb) {
            mx0 = fmaxf(mx0, fmaxf(s[nb][0], s[nb][1]));
            mx1 = fmaxf(mx1, fmaxf(s[nb][2], s[nb][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // running maxima are kept in the scaled base-2 domain (sl2 > 0 keeps the order)
        const float n0 = fmaxf(m0, mx0 * sl2), n1 = fmaxf(m1, mx1 * sl2);
        const float al0 = n0 == -INFINITY ? 1.0f : exp2f(m0 - n0);
        const float al1 = n1 == -INFINITY ? 1.0f : exp2f(m1 - n1);
        m0 = n0;
        m1 = n1;
        const float z0 = n0 == -INFINITY ? 0.0f : n0, z1 = n1 == -INFINITY ? 0.0f : n1;
        float r0 = 0.f, r1 = 0.f, e0 = 0.f, e1 = 0.f;
#pragma unroll
        for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = exp2f(fmaf(s[nb][e], sl2, -(e < 2 ? z0 : z1)));   // masked: exp2(-inf) = 0
                const float pr = __bfloat162float(__float2bfloat16_rn(p));
                s[nb][e] = pr;                       // the weight the PV product uses
                if (e < 2) { r0 += pr; e0 += p; } else { r1 += pr; e1 += p; }
            }
        }
        lr0 = lr0 * al0 + r0;
        lr1 = lr1 * al1 + r1;
        le0 = le0 * al0 + e0;
        le1 = le1 * al1 + e1;
        if (!__all_sync(0xffffffffu, al0 == 1.0f && al1 == 1.0f)) {
#pragma unroll
            for (int i = 0; i < kND; ++i) {
                o[i][0] *= al0; o[i][1] *= al0;
                o[i][2] *= al1; o[i][3] *= al1;
            }
        }
        // ---- O += P V (V = the same key rows)
        {
            const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                // A fragment order: a0 (g, k lo), a1 (g+8, k lo), a2 (g, k hi), a3 (g+8, k hi)
                const uint32_t af[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]), pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                                        pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                                        pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
                const int key = kk * 16 + rr + (mi & 1) * 8;
#pragma unroll
                for (int ndp = 0; ndp < kND / 2; ++ndp) {
                    const int piece = ndp * 2 + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(kbase + key * D * 2 + ((piece ^ (key & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(o[2 * ndp], af, b0, b1);
                    mma_bf16(o[2 * ndp + 1], af, b2, b3);
                }
            }
        }
    }
    cp_async_wait<0>();

    // ---- publish this CTA's partial state
    lr0 += __shfl_xor_sync(0xffffffffu, lr0, 1);
    lr0 += __shfl_xor_sync(0xffffffffu, lr0, 2);
    lr1 += __shfl_xor_sync(0xffffffffu, lr1, 1);
    lr1 += __shfl_xor_sync(0xffffffffu, lr1, 2);
    le0 += __shfl_xor_sync(0xffffffffu, le0, 1);
    le0 += __shfl_xor_sync(0xffffffffu, le0, 2);
    le1 += __shfl_xor_sync(0xffffffffu, le1, 1);
    le1 += __shfl_xor_sync(0xffffffffu, le1, 2);
    __syncthreads();    // every warp is done reading the key ring
#pragma unroll
    for (int i = 0; i < kND; ++i) {
        *reinterpret_cast<float2*>(sO + (h0 + g) * kOS + i * 8 + 2 * tq) = make_float2(o[i][0], o[i][1]);
        *reinterpret_cast<float2*>(sO + (h0 + g + 8) * kOS + i * 8 + 2 * tq) = make_float2(o[i][2], o[i][3]);
    }
    if (tq == 0) {
        sSt[h0 + g] = RowState{m0, lr0, le0};
        sSt[h0 + g + 8] = RowState{m1, lr1, le1};
    }
    cluster.sync();

    // ---- merge: this CTA finalises heads [rank * H / C, (rank + 1) * H / C)
    const int hpc = H / C;
    for (int it = tid; it < hpc * (D / 4); it += kThreads) {
        const int hl = it / (D / 4), d4 = it - hl * (D / 4);
        const int h = rank * hpc + hl;
        // every peer's state and slice is requested before any is combined
        RowState st[16];
        float4 v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            if (c < C) {
                st[c] = cluster.map_shared_rank(sSt, c)[h];
                v[c] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(sO, c) + h * kOS + d4 * 4);
            } else {
                st[c] = RowState{-INFINITY, 0.f, 0.f};
                v[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < 16; ++c) M = fmaxf(M, st[c].m);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float lr = 0.f, le = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float w = st[c].m == -INFINITY ? 0.0f : exp2f(st[c].m - M);
            acc.x = fmaf(w, v[c].x, acc.x);
            acc.y = fmaf(w, v[c].y, acc.y);
            acc.z = fmaf(w, v[c].z, acc.z);
            acc.w = fmaf(w, v[c].w, acc.w);
            lr = fmaf(w, st[c].lr, lr);
            le = fmaf(w, st[c].le, le);
        }
        const float inv = lr > 0.f ? 1.0f / lr : 0.0f;
        T16* out = static_cast<T16*>(a.out) + ((size_t)row * H + h) * D + d4 * 4;
        __nv_bfloat162 w0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        __nv_bfloat162 w1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&w0);
        pk.y = *reinterpret_cast<uint32_t*>(&w1);
        *reinterpret_cast<uint2*>(out) = pk;
        if (a.lse_out && d4 == 0)
            a.lse_out[(size_t)row * H + h] = le > 0.f ? (M + log2f(le)) / kLog2e : -INFINITY;
    }
    cluster.sync();     // keep this CTA's shared memory alive until every peer has read it
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Upper bound on one row's virtual keys.
long max_keys(const AttnArgs& a) {
    const long comp = a.dense ? a.N_cap : a.topk;
    const long win = a.window > 0 ? std::min<long>(a.window, a.L_raw) : 0;
    return comp + win;
}

// Cluster size: the largest power of two (<= 16, <= H/4 so every CTA merges
// at least four heads) whose rows x C CTAs still fit one wave and leave each
// CTA at least one full tile.
int choose_cluster(const AttnArgs& a) {
    const long rows = (long)a.B * a.n_q;
    const long T = max_keys(a);
    const long slots = (long)num_sms() * (a.H <= 64 ? 3 : 1);
    int C = 1;
    while (2 * C <= 16 && 2 * C <= a.H / 4 && rows * 2 * C <= slots && (T + 2 * C - 1) / (2 * C) >= kBN) C *= 2;
    return C;
}

int chunk_cap(const AttnArgs& a, int C) {
    const long T = max_keys(a);
    const long ch = ((T + C - 1) / C + kBN - 1) / kBN * kBN;
    return (int)std::max<long>(ch, kBN);
}

template <int H, int D>
cudaError_t launch_hd(const AttnArgs& a, cudaStream_t s) {
    const int C = choose_cluster(a);
    const int max_chunk = chunk_cap(a, C);
    const size_t smem = Plan<D>::kRingBytes + (size_t)H * D * 2 + sizeof(RowState) * H + sizeof(int) * max_chunk +
                        sizeof(uint32_t) * (max_chunk / 32);
    auto kern = attn_split_kernel<H, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (C > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)(a.B * a.n_q), 1);
    cfg.blockDim = dim3(H * 2, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a, max_chunk);
    count_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, cudaStream_t s) {
    switch (a.H) {
        case 16: return launch_hd<16, D>(a, s);
        case 32: return launch_hd<32, D>(a, s);
        case 64: return launch_hd<64, D>(a, s);
        case 128: return launch_hd<128, D>(a, s);
    }
    return cudaErrorNotSupported;
}

}  // namespace

bool attention_split_supported(const AttnArgs& a) {
    if (a.dt != DT_BF16 || (a.D != 64 && a.D != 128)) return false;
    if (a.H != 16 && a.H != 32 && a.H != 64 && a.H != 128) return false;
    if (a.B * (long)a.n_q > 65535) return false;
    return chunk_cap(a, choose_cluster(a)) <= kMaxChunk;
}

cudaError_t launch_attention_split(const AttnArgs& a, cudaStream_t s) {
    return a.D == 64 ? launch_d<64>(a, s) : launch_d<128>(a, s);
}

}  // namespace csa
