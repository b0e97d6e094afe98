// indexer_topk.cu -- stage 2: Lightning-Indexer score + fused causal top-k.
//
// score[t, s] = sum_h w[t, h] ReLU(qI[t, h] . kI[s]),  s < V(t) = min(floor((t+1)/m), n_entries)
//               (w: gate weights of any sign, 1 when none are given)
// idx[t, :]   = the topk largest scores, equal scores lowest index first, -1 padded
// ("百万上下文从「奢侈品」变「日用品」…" §3.2 indexer score + torch.topk, §8.2
//  streaming selection; "DS-V4 分析&学习" §1.2, §4 low-precision indexer QK.)
//
// One CTA owns one query row.  It scores the row's visible entries into
// shared memory (never global memory) as order-preserving 32-bit images of
// the fp32 scores (score_key); a four-digit MSB-first radix
// select finds the exact k-th largest key K and how many keys equal to K
// are needed; a block-wide ordered scan then writes every entry with key > K
// and the lowest-index entries with key == K.  Rows with V <= topk skip the
// scoring and write 0..V-1 followed by -1.
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxHeads = 16;
constexpr int kMaxDim = 256;

struct SelectShared {
    unsigned hist[256];
    unsigned warp_tot[2][kWarps];
    unsigned digit, rank;
};

// Loads 8 consecutive elements of a key row as fp32.
template <int KD>
__device__ __forceinline__ void load8(const void* row, int c, float* v);
template <>
__device__ __forceinline__ void load8<DT_F32>(const void* row, int c, float* v) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + c);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<DT_BF16>(const void* row, int c, float* v) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(row) + c));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
template <>
__device__ __forceinline__ void load8<DT_E4M3>(const void* row, int c, float* v) {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(row) + c));
    const uint8_t* b = reinterpret_cast<const uint8_t*>(&u);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = e4m3_value(b[i]);
}

template <int KD>
__device__ __forceinline__ size_t elem_bytes() { return KD == DT_F32 ? 4 : (KD == DT_BF16 ? 2 : 1); }

// Q modes: the query row as held in shared memory is always fp32 values `qv`
// with one multiplier per head `qs`: the fp8 scale (1 unless fp8) times the
// head's gate weight (1 without weights).
template <int QD, int KD>
__global__ void __launch_bounds__(kThreads) indexer_topk_kernel(IndexerArgs a) {
    extern __shared__ unsigned keys[];   // [N_cap] score keys of this row
    __shared__ float qv[kMaxHeads * kMaxDim];
    __shared__ float qs[kMaxHeads];
    __shared__ SelectShared sh;

    const int row = blockIdx.x;                 // b * n_q + q
    const int b = row / a.n_q;
    const int H = a.H_I, d = a.d_I, topk = a.topk;
    int* out = a.idx_out + (size_t)row * topk;
    const int t = a.q_pos ? a.q_pos[row] : a.pos0 + (row - b * a.n_q);
    const int ne = clampi(a.n_entries ? a.n_entries[b] : a.N_cap, 0, a.N_cap);
    const int V = t < 0 ? 0 : min((t + 1) / a.m, ne);

    if (V <= topk) {
        for (int j = threadIdx.x; j < topk; j += kThreads) out[j] = j < V ? j : -1;
        return;
    }

    // ---- the query row (fp8: quantise per head in fp32 unless given codes)
    if constexpr (QD == DT_E4M3) {
        const uint8_t* src = static_cast<const uint8_t*>(a.qI) + (size_t)row * H * d;
        for (int p = threadIdx.x; p < H * d; p += kThreads) qv[p] = e4m3_value(src[p]);
        for (int h = threadIdx.x; h < H; h += kThreads) qs[h] = a.qI_scale[(size_t)row * H + h];
    } else if constexpr (KD == DT_E4M3) {   // bf16 query quantised in the kernel
        const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(a.qI) + (size_t)row * H * d;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int h = warp; h < H; h += kWarps) {
            float amax = 0.0f;
            for (int c = lane; c < d; c += 32) amax = fmaxf(amax, fabsf(__bfloat162float(src[h * d + c])));
            for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
            for (int c = lane; c < d; c += 32)
                qv[h * d + c] = e4m3_value(e4m3_code(__fdiv_rn(__bfloat162float(src[h * d + c]), scale)));
            if (lane == 0) qs[h] = scale;
        }
    } else {
        using TQ = typename std::conditional<QD == DT_F32, float, __nv_bfloat16>::type;
        const TQ* src = static_cast<const TQ*>(a.qI) + (size_t)row * H * d;
        for (int p = threadIdx.x; p < H * d; p += kThreads) qv[p] = to_f32(src[p]);
        for (int h = threadIdx.x; h < H; h += kThreads) qs[h] = 1.0f;
    }
    __syncthreads();
    if (a.qI_weight) {
        for (int h = threadIdx.x; h < H; h += kThreads) qs[h] *= a.qI_weight[(size_t)row * H + h];
        __syncthreads();
    }

    // ---- scores of the visible entries, as order-preserving keys
    const uint8_t* kbase = static_cast<const uint8_t*>(a.kI);   // rows from cache_row()
    for (int s = threadIdx.x; s < V; s += kThreads) {
        const long crow = cache_row(a.pages, a.N_cap, b, s);
        if (crow < 0) {                      // page outside the pool: an absent (zero) row
            keys[s] = score_key(0.0f);
            continue;
        }
        const void* krow = kbase + (size_t)crow * d * elem_bytes<KD>();
        float dots[kMaxHeads];
#pragma unroll
        for (int h = 0; h < kMaxHeads; ++h) dots[h] = 0.0f;
        for (int c = 0; c < d; c += 8) {
            float kv8[8];
            load8<KD>(krow, c, kv8);
#pragma unroll
            for (int h = 0; h < kMaxHeads; ++h) {
                if (h < H) {
                    const float* qh = qv + h * d + c;
#pragma unroll
                    for (int i = 0; i < 8; ++i) dots[h] = fmaf(qh[i], kv8[i], dots[h]);
                }
            }
        }
        float sc = 0.0f;
#pragma unroll
        for (int h = 0; h < kMaxHeads; ++h)
            if (h < H) sc = fmaf(qs[h], relu0(dots[h]), sc);
        if constexpr (KD == DT_E4M3) sc *= a.kI_scale[crow];
        keys[s] = score_key(sc);
    }
    __syncthreads();

    // ---- radix select: exact k-th largest key K, and how many == K to take
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned prefix = 0, pmask = 0, rank = (unsigned)topk;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int s = threadIdx.x; s < V; s += kThreads) {
            const unsigned k = keys[s];
            if ((k & pmask) == prefix) atomicAdd(&sh.hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns digits 255-8l .. 248-8l (descending)
            unsigned c[8], tot = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) { c[i] = sh.hist[255 - 8 * lane - i]; tot += c[i]; }
            unsigned incl = tot;   // inclusive prefix over lanes (higher digits first)
            for (int off = 1; off < 32; off <<= 1) {
                unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const unsigned excl = incl - tot;
            const bool mine = excl < rank && rank <= incl;
            if (mine) {
                unsigned run = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (run < rank && rank <= run + c[i]) {
                        sh.digit = 255u - 8u * lane - i;
                        sh.rank = rank - run;
                    }
                    run += c[i];
                }
            }
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        pmask |= 255u << shift;
        rank = sh.rank;
        __syncthreads();
    }
    const unsigned K = prefix;
    const unsigned need_eq = rank;              // >= 1 keys equal to K are taken
    const unsigned n_gt = (unsigned)topk - need_eq;

    // ---- ordered emission: keys > K at [0, n_gt), first need_eq keys == K after
    unsigned run_gt = 0, run_eq = 0;
    for (int base = 0; base < V; base += kThreads) {
        const int s = base + threadIdx.x;
        const unsigned k = s < V ? keys[s] : 0u;
        const bool gt = s < V && k > K;
        const bool eq = s < V && k == K;
        const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
        const unsigned lt_mask = (1u << lane) - 1u;
        if (lane == 0) { sh.warp_tot[0][warp] = __popc(bg); sh.warp_tot[1][warp] = __popc(be); }
        __syncthreads();
        unsigned off_g = 0, off_e = 0, tot_g = 0, tot_e = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            if (w < warp) { off_g += sh.warp_tot[0][w]; off_e += sh.warp_tot[1][w]; }
            tot_g += sh.warp_tot[0][w];
            tot_e += sh.warp_tot[1][w];
        }
        if (gt) {
            const unsigned r = run_gt + off_g + __popc(bg & lt_mask);
            if (r < n_gt) out[r] = s;
        }
        if (eq) {
            const unsigned r = run_eq + off_e + __popc(be & lt_mask);
            if (r < need_eq) out[n_gt + r] = s;
        }
        run_gt += tot_g;
        run_eq += tot_e;
        __syncthreads();
    }
}

template <int QD, int KD>
cudaError_t launch_t(const IndexerArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(unsigned) * (size_t)a.N_cap;
    auto kern = indexer_topk_kernel<QD, KD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.n_q), kThreads, smem, s>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer_packed(const IndexerArgs& a, int max_entries, cudaStream_t s) {
    IndexerArgs shape = a;             // the per-sequence shape decides the kernel
    shape.N_cap = max_entries;
    if (a.vl == nullptr || a.pages.bt != nullptr || !indexer_tc_supported(shape))
        return cudaErrorNotSupported;
    uint32_t* err = device_error_word();
    if (!err) return cudaErrorUnknown;
    return launch_indexer_tc(a, err, s);
}

cudaError_t launch_indexer_topk(const IndexerArgs& a, cudaStream_t s, const char** why) {
    if (a.B <= 0 || a.n_q <= 0) return cudaSuccess;
    if (a.H_I > kMaxHeads || a.d_I > kMaxDim) {
        *why = "csa_indexer_topk: H_I > 16 or d_I > 256";
        return cudaErrorNotSupported;
    }
    if (a.pages.bt == nullptr && indexer_tc_supported(a)) {     // paged caches: decode kernels
        uint32_t* err = device_error_word();
        if (!err) return cudaErrorUnknown;
        return launch_indexer_tc(a, err, s);
    }
    if (indexer_split_supported(a)) return launch_indexer_split(a, s);
    if (a.N_cap > 40960) {      // one row's score keys must fit the CTA's shared memory
        *why = "csa_indexer_topk: N_cap > 40960 needs fp8 keys with scales, d_I in {64, 128}, H_I <= 8";
        return cudaErrorNotSupported;
    }
    if (a.qI_dt == DT_F32 && a.kI_dt == DT_F32) return launch_t<DT_F32, DT_F32>(a, s);
    if (a.qI_dt == DT_BF16 && a.kI_dt == DT_BF16) return launch_t<DT_BF16, DT_BF16>(a, s);
    if (a.qI_dt == DT_BF16 && a.kI_dt == DT_E4M3) return launch_t<DT_BF16, DT_E4M3>(a, s);
    if (a.qI_dt == DT_E4M3 && a.kI_dt == DT_E4M3) return launch_t<DT_E4M3, DT_E4M3>(a, s);
    // rotated keys against query codes that the caller rotated: plain fp8 scoring
    if (a.qI_dt == DT_E4M3 && a.kI_dt == DT_E4M3H) return launch_t<DT_E4M3, DT_E4M3>(a, s);
    if (a.kI_dt == DT_E4M3H) {
        *why = "csa_indexer_topk: Hadamard keys with bf16 queries need d_I 64 (or 128 with few rows)";
        return cudaErrorNotSupported;
    }
    *why = "csa_indexer_topk: unsupported (qI_dt, kI_dt) pair";
    return cudaErrorNotSupported;
}

}  // namespace csa
