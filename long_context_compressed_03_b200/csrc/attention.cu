// attention.cu -- stage 3: joint-softmax shared-KV MQA over the selected
// compressed entries (CSA) or all visible entries (HCA) plus the sliding
// window of raw rows.
//
// For query row (b, q) at position t, head h:
//   keys = compressed set ∪ { raw row j : raw_pos0[b]+j in [max(0, t-W+1), t] }
//   o = sum_s softmax_s(scale * q.key_s) key_s      (key = value, one KV head)
// ("DS-V4 分析&学习" §1.2, §1.4, §1.5; "百万上下文从「奢侈品」变「日用品」…"
//  §4.3, §5.2 window [max(0,i-W+1), i] and 1/sqrt(head_dim).)
//
// Generic path: one CTA per query row and all H heads (MQA: every head reads
// the same key block, staged once in shared memory as fp32).  Keys stream in
// blocks of 32 through an online (running max / running sum) softmax kept
// in base 2; the compressed part and the window part are one sequence of
// "virtual" keys so both share a single softmax.
#include <math.h>

#include "attn_rows.cuh"
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kBK = 32;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int H, int D>
__global__ void __launch_bounds__(kThreads) attn_generic_kernel(AttnArgs a) {
    constexpr int TPH = kThreads / H;    // threads per head
    constexpr int KPT = kBK / TPH;       // keys per thread in the score step
    constexpr int DPT = D / TPH;         // output dims per thread
    constexpr int DP = D + 1;            // padded row stride (bank spread)
    extern __shared__ float sm[];
    float* Qs = sm;                      // [H][DP]
    float* Ks = Qs + H * DP;             // [kBK][DP]
    float* Ps = Ks + kBK * DP;           // [H][kBK]
    int* valid = reinterpret_cast<int*>(Ps + H * kBK);   // [kBK]
    const T** krow = reinterpret_cast<const T**>(valid + kBK);  // [kBK]

    const int row = blockIdx.x;
    const int b = row / a.n_q;
    const int t = a.q_pos ? a.q_pos[row] : a.pos0 + (row - b * a.n_q);
    const RowKeys rk = row_keys(a, b, t);
    const int total = rk.n_comp + rk.n_win;

    const T* q = static_cast<const T*>(a.q) + (size_t)row * H * D;
    const T* kvc = static_cast<const T*>(a.kv_c);          // rows from cache_row()
    const T* kvr = static_cast<const T*>(a.kv_raw) + (size_t)b * a.L_raw * D;
    const float qscale = a.scale * kLog2e;
    for (int p = threadIdx.x; p < H * D; p += kThreads) {
        const int h = p / D, c = p - h * D;
        Qs[h * DP + c] = to_f32(q[p]) * qscale;
    }

    const int h = threadIdx.x / TPH, sub = threadIdx.x % TPH;
    float o[DPT];
#pragma unroll
    for (int i = 0; i < DPT; ++i) o[i] = 0.0f;
    float mrun = -INFINITY, lrun = 0.0f;

    for (int base = 0; base < total; base += kBK) {
        __syncthreads();
        if (threadIdx.x < kBK) {
            const int kk = base + threadIdx.x;
            const T* ptr = nullptr;
            if (kk < rk.n_comp) {
                const int s = a.dense ? kk : a.idx[(size_t)row * a.topk + kk];
                if (s >= 0 && s < a.N_cap) {
                    const long r = cache_row(a.pages, a.N_cap, b, s);
                    if (r >= 0) ptr = kvc + (size_t)r * D;
                }
            } else if (kk < total) {
                ptr = kvr + (size_t)(rk.win_lo + kk - rk.n_comp) * D;
            }
            krow[threadIdx.x] = ptr;
            valid[threadIdx.x] = ptr != nullptr;
        }
        __syncthreads();
        for (int p = threadIdx.x; p < kBK * D; p += kThreads) {
            const int j = p / D, c = p - j * D;
            const T* ptr = krow[j];
            Ks[j * DP + c] = ptr ? to_f32(ptr[c]) : 0.0f;
        }
        __syncthreads();

        // scores of this thread's keys for head h (base-2 domain)
        float sc[KPT];
        float bmax = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < KPT; ++jj) {
            const int j = sub * KPT + jj;
            float acc = 0.0f;
            const float* qh = Qs + h * DP;
            const float* kj = Ks + j * DP;
            for (int c = 0; c < D; ++c) acc = fmaf(qh[c], kj[c], acc);
            sc[jj] = valid[j] ? acc : -INFINITY;
            bmax = fmaxf(bmax, sc[jj]);
        }
        for (int off = TPH / 2; off; off >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
        const float mnew = fmaxf(mrun, bmax);
        const float alpha = (mnew == -INFINITY) ? 1.0f : exp2f(mrun - mnew);
        float psum = 0.0f;
#pragma unroll
        for (int jj = 0; jj < KPT; ++jj) {
            const float p = (sc[jj] == -INFINITY) ? 0.0f : exp2f(sc[jj] - mnew);
            Ps[h * kBK + sub * KPT + jj] = p;
            psum += p;
        }
        for (int off = TPH / 2; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        lrun = lrun * alpha + psum;
        mrun = mnew;
#pragma unroll
        for (int i = 0; i < DPT; ++i) o[i] *= alpha;
        __syncthreads();
        for (int j = 0; j < kBK; ++j) {
            const float p = Ps[h * kBK + j];
            const float* kj = Ks + j * DP;
#pragma unroll
            for (int i = 0; i < DPT; ++i) o[i] = fmaf(p, kj[i * TPH + sub], o[i]);
        }
    }

    T* out = static_cast<T*>(a.out) + (size_t)row * H * D + (size_t)h * D;
    const float inv = lrun > 0.0f ? 1.0f / lrun : 0.0f;
#pragma unroll
    for (int i = 0; i < DPT; ++i) store_out<T>(out + i * TPH + sub, o[i] * inv);
    if (a.lse_out && sub == 0)
        a.lse_out[(size_t)row * H + h] = lrun > 0.0f ? (mrun + log2f(lrun)) / kLog2e : -INFINITY;
}

template <typename T, int H, int D>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
    const int DP = D + 1;
    const size_t smem = sizeof(float) * ((size_t)H * DP + (size_t)kBK * DP + (size_t)H * kBK) +
                        sizeof(int) * kBK + sizeof(void*) * kBK;
    auto kern = attn_generic_kernel<T, H, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.B * a.n_q), kThreads, smem, s>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_heads(const AttnArgs& a, cudaStream_t s, const char** why) {
    switch (a.H) {
        case 8: return launch_t<T, 8, D>(a, s);
        case 16: return launch_t<T, 16, D>(a, s);
        case 32: return launch_t<T, 32, D>(a, s);
        case 64: return launch_t<T, 64, D>(a, s);
        case 128: return launch_t<T, 128, D>(a, s);
    }
    *why = "attention: H must be one of 8, 16, 32, 64, 128";
    return cudaErrorNotSupported;
}

template <typename T>
cudaError_t launch_dims(const AttnArgs& a, cudaStream_t s, const char** why) {
    if (a.D == 64) return launch_heads<T, 64>(a, s, why);
    if (a.D == 128) return launch_heads<T, 128>(a, s, why);
    *why = "attention: D must be 64 or 128";
    return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_attention_packed(const AttnArgs& a, cudaStream_t s) {
    if (a.vl == nullptr || a.pages.bt != nullptr || !attention_tc_supported(a))
        return cudaErrorNotSupported;
    uint32_t* err = device_error_word();
    if (!err) return cudaErrorUnknown;
    return launch_attention_tc(a, err, s);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s, const char** why) {
    if (a.B <= 0 || a.n_q <= 0) return cudaSuccess;
    if (a.pages.bt == nullptr && attention_tc_supported(a)) {   // paged caches: decode kernels
        uint32_t* err = device_error_word();
        if (!err) return cudaErrorUnknown;
        return launch_attention_tc(a, err, s);
    }
    if (attention_dec_tc_supported(a)) {
        uint32_t* err = device_error_word();
        if (!err) return cudaErrorUnknown;
        return launch_attention_dec_tc(a, err, s);
    }
    if (attention_split_supported(a)) return launch_attention_split(a, s);
    if (a.dt == DT_F32) return launch_dims<float>(a, s, why);
    if (a.dt == DT_BF16) return launch_dims<__nv_bfloat16>(a, s, why);
    *why = "attention: dt must be F32 or BF16";
    return cudaErrorNotSupported;
}

}  // namespace csa
