// attention_dec_tc.cu -- stage 3 for decode rows on the tensor cores (tcgen05):
// one query row's 64 heads x 128 dims against a share of its keys, with the
// shares of a thread-block cluster merged through distributed shared memory.
//
// For query row (b, q) at position t and head h (one shared K = V head):
//   o[h] = sum_s softmax_s(scale * q[h] . key_s) key_s
// over the multiset {selected or visible compressed entries} ∪ {window rows}
// ("DS-V4 分析&学习" §1.2 joint softmax over compressed + window keys, §1.4
//  HCA over every visible entry; "百万上下文从「奢侈品」变「日用品」…" §4.3 window
//  [max(0, t-W+1), t], §5.2 1/sqrt(head_dim)).
//
// A decode row has 64 heads but thousands of keys, so the score tile is taken
// transposed: S^T = K Q^T with the 128 keys of a tile as the M = 128 rows of
// the tensor core and the 64 heads as N.  Every TMEM lane then holds one key's
// 64 scores, and the softmax threads (one key each) keep every lane busy.
// Row r's virtual key list (compressed part, then window part) is cut into
// 128-key tiles dealt round-robin to the C CTAs of a cluster (the window tiles
// of a CTA first, so the first tiles need no row codes).  A CTA:
//   * stages its share's row codes (entry, raw row or none) in shared memory;
//   * loader warps stream 128-key tiles through a 4-stage ring into the
//     128-byte-swizzled layout the tensor core reads.  The compressed part of
//     the key list is padded (with masked keys) to whole tiles, so a tile is
//     either entries or window rows: contiguous tiles (HCA entries, the
//     window) come by two TMA box loads of 128 rows, gathered ones (CSA
//     entries by index, paged caches) by 16-byte cp.async;
//   * S^T = K Q^T (M = 128, N = 64, K = 128) into one of two TMEM buffers, so
//     the next tile's product runs while a tile's softmax does;
//   * the softmax warps write P^T (key-major, bf16) to shared memory and
//     O += P V (M = 64 heads, N = 128, K = 128 keys) accumulates in TMEM, P
//     read as an MN-major operand and V the key tile read MN-major;
//   * each softmax thread adds its key's weights into per-head registers (the
//     bf16-rounded ones the product used, l_r, and the exact ones, l_e, for
//     the log-sum-exp); one transposing warp reduction at the end sums them;
//   * pushes (offset m, l_r, l_e, unnormalised O) of every head over DSMEM
//     to the CTA of the cluster that finalises it; after a cluster barrier
//     CTA c merges its range of heads from its inbox and writes o and the
//     log-sum-exp.
// The offset m of a head is a whole number: set from the head's first keys
// and raised by whole steps only when a weight would exceed 2^15, so every
// rescale (of O in TMEM and of the sums) is an exact power of two.  O is
// normalised by l_r, the sum of the bf16-rounded weights the products used.
// Roles (21 warps): warps 0-3 load; warps 4-19 run the softmax (warp w reads
// TMEM lanes 32 (w % 4) .. +31, i.e. keys, and heads 16 ((w - 4) / 4) .. +15);
// warp 20 allocates TMEM and one lane issues every MMA.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>
#include <limits.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "attn_rows.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace cg = cooperative_groups;

namespace csa {
namespace {

using namespace tc;

constexpr int kH = 64;
constexpr int kD = 128;
constexpr int kBN = 128;                     // keys per tile (the MMA's M)
constexpr int kStages = 4;                   // key ring depth (a fifth stage measured no faster)
constexpr int kLoadWarps = 4;
constexpr int kSoftWarps = 16;
constexpr int kMmaWarp = kLoadWarps + kSoftWarps;
constexpr int kLoadThreads = kLoadWarps * 32;
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kHPT = 16;                     // heads per softmax thread
constexpr int kTileBytes = kBN * kD * 2;     // 32 KB: two 64-dim halves of 128 rows x 128 B
constexpr int kHalfK = kBN * 128;            // one 64-dim half of a tile
constexpr int kHalfQ = kH * 128;             // one 64-dim half of Q
constexpr int kPBytes = kBN * kH * 2;        // P^T: 128 keys x 64 heads, bf16
constexpr int kMaxChunk = 4096;              // keys per CTA (row codes in shared memory)
constexpr int kOS = kD + 4;                  // fp32 partial-O row stride (floats)
constexpr int kMaxParts = 80;                // >= C * ceil(64 / C) for every C <= 16
constexpr int kBarSoft = 1;                  // named barrier of the softmax warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kHeadLog2 = 15.0f;           // largest log2 weight before the offset is raised
constexpr int kRaiseTo = 8;                  // after a raise the tile's largest is in (7, 8]
static_assert(kLoadThreads == kBN, "one loader thread per key row of a tile");
static_assert(kSoftThreads == 4 * kBN && 4 * kHPT == kH, "four softmax threads per key, 16 heads each");

struct __align__(8) Ctrl {
    uint64_t full[kStages];      // the tile landed (one arrival per loader thread, plus TMA bytes)
    uint64_t freeb[kStages];     // the tile's P.V completed
    uint64_t s_full[2];          // S buffer holds the tile's product
    uint64_t p_ready[2];         // P buffer written (one arrival per softmax warp)
    uint64_t p_free[2];          // P buffer read by its P.V
    uint64_t pv_done;            // one phase per P.V
    uint64_t o_done;             // the last P.V completed (one phase)
    uint64_t fin;
    uint64_t stall_bar;          // test hook: a barrier nothing completes
    uint32_t tmem_base;
    int abort;
};
struct RowState {
    float m, lr, le;
};

// Shared memory: Q, key ring, P buffers, control, per-head offsets, scales and
// tile maxima, partial sums, the merge inbox of states and row codes.  After
// the last tile the ring holds the merge inbox of partial O rows.
struct DecSmem {
    size_t q, ring, p, ctrl, m, alpha, tmax, lsum, st, rows, bytes;
};
__host__ __device__ inline DecSmem dec_smem(int max_chunk) {
    DecSmem s;
    s.q = 0;
    s.ring = s.q + kH * kD * 2;
    s.p = s.ring + (size_t)kStages * kTileBytes;
    s.ctrl = s.p + 2 * (size_t)kPBytes;
    s.m = s.ctrl + ((sizeof(Ctrl) + 15) & ~(size_t)15);
    s.alpha = s.m + kH * 4;
    s.tmax = s.alpha + kH * 4;
    s.lsum = s.tmax + kH * 4;                     // [2][4][64] floats: l_r, l_e per lane quarter
    s.st = s.lsum + 2 * 4 * kH * 4;
    s.rows = s.st + ((kMaxParts * sizeof(RowState) + 15) & ~(size_t)15);
    s.bytes = s.rows + (size_t)max_chunk * 4 + 1024;   // + alignment slack
    return s;
}
static_assert(kMaxParts * kOS * 4 <= kStages * kTileBytes, "the merge inbox fits the key ring");

// Add tx bytes the current phase of the barrier waits for (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// 2^k for a whole number k <= 0 (0 below the normal range)
__device__ __forceinline__ float exp2_int(int k) {
    return k < -126 ? 0.0f : __int_as_float((127 + k) << 23);
}
__device__ __forceinline__ uint32_t bf2(float lo, float hi, float& rlo, float& rhi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    const float2 r = __bfloat1622float2(h);
    rlo = r.x;
    rhi = r.y;
    return *reinterpret_cast<const uint32_t*>(&h);
}
// OR of pred over the `count` threads of named barrier `id` (all of them arrive).
__device__ __forceinline__ bool bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// byte offset of 16-byte chunk c (0..15) of row r in a 128-byte-swizzled tile
// of two 64-column halves, half_bytes apart
__device__ __forceinline__ uint32_t sw_chunk(int r, int c, int half_bytes) {
    return (uint32_t)((c >> 3) * half_bytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Sum of v[i] over the 32 lanes of the warp for every i < 16; lanes L and
// L + 16 return the total of index L (halving exchanges, then one more add).
__device__ __forceinline__ float warp_transpose_sum16(float (&v)[kHPT], int lane) {
#pragma unroll
    for (int o = kHPT / 2; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The CTA of a C-CTA cluster that finalises head h: heads [c 64 / C, (c + 1) 64 / C).
__device__ __forceinline__ int owner_of(int h, int C) { return ((h + 1) * C + kH - 1) / kH - 1; }

// tm_c: the compressed cache as [B * N_cap, 128] rows, tm_w: the window
// cache as [B * L_raw, 128] rows, both with boxes of {64, 128} (tm_c unused
// when the compressed cache is paged or gathered by index).
template <bool LSE>
__global__ void __launch_bounds__(kThreads, 1) attn_dec_tc_kernel(const __grid_constant__ CUtensorMap tm_c,
                                                                 const __grid_constant__ CUtensorMap tm_w,
                                                                 AttnArgs a, int max_chunk, uint32_t* err,
                                                                 uint64_t wait_ns, int stall) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const DecSmem L = dec_smem(max_chunk);
    uint8_t* sQ = base + L.q;
    uint8_t* ring = base + L.ring;
    uint8_t* sP = base + L.p;
    Ctrl* ctl = reinterpret_cast<Ctrl*>(base + L.ctrl);
    float* sM = reinterpret_cast<float*>(base + L.m);
    float* sAlpha = reinterpret_cast<float*>(base + L.alpha);
    int* sTmax = reinterpret_cast<int*>(base + L.tmax);
    float* sLsum = reinterpret_cast<float*>(base + L.lsum);
    RowState* sIn = reinterpret_cast<RowState*>(base + L.st);     // merge inbox: states
    int* sRow = reinterpret_cast<int*>(base + L.rows);
    float* sInO = reinterpret_cast<float*>(ring);                  // merge inbox: partial O rows

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int b = row / a.n_q;
    const int t = a.q_pos ? a.q_pos[row] : a.pos0 + (row - b * a.n_q);
    const RowKeys rk = row_keys(a, b, t);
    const int cpad = (rk.n_comp + kBN - 1) / kBN * kBN;     // window keys start on a tile
    const int T = cpad + rk.n_win;
    const int NT = (T + kBN - 1) / kBN;                     // tiles of the row
    const int ntile = rank < NT ? (NT - rank + C - 1) / C : 0;
    // this CTA's tile j is the row's tile rank + (ntile - 1 - j) C: the window tiles first
    auto kk0_of = [&](int j) { return (rank + (ntile - 1 - j) * C) * kBN; };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &ctl->abort;
    const float sl2 = a.scale * kLog2e;
    const int hmax = (kH + C - 1) / C;                      // heads a CTA finalises, at most
    const bool paged = a.pages.bt != nullptr;
    const int lead = min(ntile, kStages - 1);              // tiles in flight before the first is consumed

    using T16 = __nv_bfloat16;
    const T16* kvc = static_cast<const T16*>(a.kv_c);
    const T16* kvr = static_cast<const T16*>(a.kv_raw) + (size_t)b * a.L_raw * kD;

    // tile j by TMA: 1 = compressed entries (dense, unpaged), 2 = window rows, 0 = gathered
    auto tile_kind = [&](int j) -> int {
        const int kk0 = kk0_of(j);
        if (kk0 >= cpad) return 2;
        return (a.dense && !paged) ? 1 : 0;
    };
    auto issue_tma = [&](int j) {
        const int kind = tile_kind(j);
        uint8_t* dst0 = ring + (j % kStages) * kTileBytes;
        uint64_t* bar = &ctl->full[j % kStages];
        const int kk0 = kk0_of(j);
        const int y = kind == 1 ? b * a.N_cap + kk0 : b * a.L_raw + rk.win_lo + (kk0 - cpad);
        const CUtensorMap* m = kind == 1 ? &tm_c : &tm_w;
        mbar_expect_tx(bar, kTileBytes);
        tma_load_2d(dst0, m, 0, y, bar);
        tma_load_2d(dst0 + kHalfK, m, 64, y, bar);
    };

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->full[s], kLoadThreads);
            mbar_init(&ctl->freeb[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->s_full[i], 1);
            mbar_init(&ctl->p_ready[i], kSoftWarps);
            mbar_init(&ctl->p_free[i], 1);
        }
        mbar_init(&ctl->pv_done, 1);
        mbar_init(&ctl->o_done, 1);
        mbar_init(&ctl->fin, 1);
        mbar_init(&ctl->stall_bar, 1);
        ctl->abort = (*reinterpret_cast<volatile uint32_t*>(err) != 0u) ? 1 : 0;
        fence_barrier_init();
    }
    if (tid < kH) {
        sM[tid] = -INFINITY;
        sTmax[tid] = INT_MIN;
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&ctl->tmem_base, 256);
        tmem_relinquish();
    }
    __syncthreads();
    // the first contiguous tiles and Q need no row codes: start them now
    // (nothing is started when an earlier launch left the error word set)
    if (tid == 0 && !*abort) {
        prefetch_tmap(&tm_c);
        prefetch_tmap(&tm_w);
        for (int j = 0; j < lead; ++j)
            if (tile_kind(j)) issue_tma(j);
    }
    if (warp < kLoadWarps) {
        const T16* q = static_cast<const T16*>(a.q) + (size_t)row * kH * kD;
#pragma unroll
        for (int i = 0; i < kH * kD * 2 / 16 / kLoadThreads; ++i) {
            const int c = tid + i * kLoadThreads;
            const int h = c >> 4, c16 = c & 15;
            cp_async16(sQ + sw_chunk(h, c16, kHalfQ), q + (size_t)h * kD + c16 * 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");          // Q: the oldest group
    }
    // The indices may come from the kernel launched just before this one (the
    // indexer lets this grid start early, see launch_attention_dec_tc): wait
    // for it before the first read of idx.  Everything above reads only the
    // caller's inputs, never a preceding kernel's output.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // ---- row codes: >= 0 physical row of a compressed entry, <= -2 raw row -(code + 2), -1 none
    for (int i = tid; i < ntile * kBN; i += kThreads) {
        const int kk = kk0_of(i / kBN) + (i % kBN);
        int code = -1;
        if (kk < T) {
            if (kk < rk.n_comp) {
                const int s = a.dense ? kk : a.idx[(size_t)row * a.topk + kk];
                code = (s >= 0 && s < a.N_cap) ? (int)cache_row(a.pages, a.N_cap, b, s) : -1;
            } else if (kk >= cpad) {
                code = -(rk.win_lo + kk - cpad) - 2;
            }
        }
        sRow[i] = code;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t t_o = tmem + 128;                 // O: TMEM columns [128, 256), M = 64 layout

    if (warp < kLoadWarps) {
        // ------------------------------------------------------------ loaders
        const int lt = tid;
        int last = -1;                                   // the last tile handed to issue_tile
        // tile j: TMA tiles were started by thread 0 (prologue) or start here,
        // and every loader arrives at once (the barrier then completes on the
        // TMA bytes; before tile 0 this loader's part of Q must have landed);
        // gathered rows by 16-byte copies, whose loaders arrive once they
        // landed.  One commit group per tile, after the group of Q.
        auto issue_tile = [&](int j, bool tma_started) {
            last = j;
            if (tile_kind(j)) {
                if (lt == 0 && !tma_started && !*abort) issue_tma(j);
                if (j == 0) {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");   // only Q is pending
                    fence_proxy_async_smem();
                }
                mbar_arrive(&ctl->full[j % kStages]);       // after thread 0's expect_tx
            } else {
                uint8_t* dst0 = ring + (j % kStages) * kTileBytes;
#pragma unroll 4
                for (int i = 0; i < kTileBytes / 16 / kLoadThreads; ++i) {
                    const int c = lt + i * kLoadThreads;          // 0 .. 2047
                    const int r = c >> 4, c16 = c & 15;
                    const int code = sRow[j * kBN + r];
                    const T16* src = code >= 0 ? kvc + (size_t)code * kD
                                               : (code <= -2 ? kvr + (size_t)(-code - 2) * kD : nullptr);
                    uint8_t* dst = dst0 + sw_chunk(r, c16, kHalfK);
                    if (src) cp_async16(dst, src + c16 * 8);
                    else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        for (int j = 0; j < lead; ++j) issue_tile(j, true);
        for (int j = 0; j < ntile; ++j) {
            if (!tile_kind(j)) {
                // tile j landed: the younger groups still pending are tiles j+1 .. min(j+2, ntile-1)
                const int younger = min(ntile - 1, j + kStages - 2) - j;
                if (younger >= 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
                else if (younger == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
                else asm volatile("cp.async.wait_group 0;" ::: "memory");
                fence_proxy_async_smem();
                mbar_arrive(&ctl->full[j % kStages]);
            }
            const int nj = j + kStages - 1;
            if (nj < ntile) {
                const int use = nj / kStages;
                if (use > 0 && !mbar_wait(&ctl->freeb[nj % kStages], (use - 1) & 1, abort, err, wait_ns)) break;
                issue_tile(nj, false);
            }
        }
        cp_async_wait_all();
        // TMA tiles still landing (an abort) land before the CTA's shared
        // memory is given up.  The last kStages tiles handed out are the
        // latest phase of each stage's barrier (so its parity is unambiguous);
        // a TMA tile's loaders arrived when it was handed out, so its phase
        // completes once its bytes land (at once if it was not started).
        if (lt == 0) {
            volatile int never = 0;
            for (int j = max(0, last - (kStages - 1)); j <= last; ++j)
                if (tile_kind(j)) mbar_wait(&ctl->full[j % kStages], (j / kStages) & 1, &never, err);
        }
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------------ softmax
        const int sw = warp - kLoadWarps;
        const int qd = warp & 3;                         // TMEM lane quarter: keys 32 qd .. +31
        const int hq = sw >> 2;                          // heads 16 hq .. +15
        const int key = 32 * qd + lane;
        const int st = tid - kLoadThreads;               // 0 .. 511
        const uint32_t t_s = tmem + ((uint32_t)(32 * qd) << 16) + kHPT * hq;
        const float* mrow = sM + kHPT * hq;
        float acc_r[kHPT], acc_e[kHPT];
#pragma unroll
        for (int i = 0; i < kHPT; ++i) {
            acc_r[i] = 0.0f;
            acc_e[i] = 0.0f;
        }
        bool ok = true;
        for (int j = 0; j < ntile; ++j) {
            bool good = mbar_wait(&ctl->s_full[j & 1], (j >> 1) & 1, abort, err, wait_ns);
            // P buffer j & 1 is free once the P.V of tile j - 2 completed
            if (good && j >= 2) good = mbar_wait(&ctl->p_free[j & 1], ((j >> 1) - 1) & 1, abort, err, wait_ns);
            good = __all_sync(0xffffffffu, good);
            tc_fence_after();
            float sv[kHPT];
            if (good) tmem_ld16(t_s + (j & 1) * 64, sv);
            const bool valid = good && sRow[j * kBN + key] != -1;
            // P = exp2(S*sl2 - m) of this key's 16 heads in bf16 pairs; does a
            // weight exceed 2^15 under the current offsets?
            uint32_t w[kHPT / 2];
            auto exp_pass = [&]() -> bool {
                bool ovf = false;
#pragma unroll
                for (int i = 0; i < kHPT; i += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(mrow + i);
                    const float x0 = fmaf(sv[i], sl2, -m4.x), x1 = fmaf(sv[i + 1], sl2, -m4.y);
                    const float x2 = fmaf(sv[i + 2], sl2, -m4.z), x3 = fmaf(sv[i + 3], sl2, -m4.w);
                    ovf |= fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)) > kHeadLog2;
                    float r0, r1;
                    w[i >> 1] = valid ? bf2(ex2(x0), ex2(x1), r0, r1) : 0u;
                    w[(i >> 1) + 1] = valid ? bf2(ex2(x2), ex2(x3), r0, r1) : 0u;
                }
                return valid && ovf;
            };
            const bool ovf = good && exp_pass();
            if (bar_or(kBarSoft, kSoftThreads, ovf || !good)) {
                if (bar_or(kBarSoft, kSoftThreads, !good)) { ok = false; break; }
                // ---- raise the offsets of the heads whose tile maximum demands it
#pragma unroll
                for (int i = 0; i < kHPT; ++i) {
                    const int v = __reduce_max_sync(0xffffffffu, valid ? (int)ceilf(sv[i] * sl2) : INT_MIN);
                    if (lane == 0) atomicMax(&sTmax[kHPT * hq + i], v);
                }
                named_sync(kBarSoft, kSoftThreads);
                if (st < kH) {
                    const int tm = sTmax[st];
                    const float mo = sM[st];
                    float alpha = 1.0f;
                    if (tm != INT_MIN && (mo == -INFINITY || (float)tm - mo > kHeadLog2)) {
                        const float mn = mo == -INFINITY ? (float)tm : (float)(tm - kRaiseTo);
                        alpha = mo == -INFINITY ? 0.0f : exp2_int((int)(mo - mn));
                        sM[st] = mn;
                    }
                    sAlpha[st] = alpha;
                    sTmax[st] = INT_MIN;
                }
                named_sync(kBarSoft, kSoftThreads);
#pragma unroll
                for (int i = 0; i < kHPT; ++i) {
                    const float al = sAlpha[kHPT * hq + i];
                    acc_r[i] *= al;
                    acc_e[i] *= al;
                }
                if (j > 0) {
                    // O holds the earlier tiles' products: the last P.V must have landed
                    const bool pv = __all_sync(0xffffffffu, mbar_wait(&ctl->pv_done, (j - 1) & 1, abort, err, wait_ns));
                    tc_fence_after();
                    if (pv) {
                        // this warp's TMEM lanes hold heads 16 qd + lane (lanes < 16); columns 32 hq .. +31
                        const float al = lane < 16 ? sAlpha[16 * qd + lane] : 1.0f;
                        const uint32_t t_row = t_o + ((uint32_t)(32 * qd) << 16) + 32 * hq;
                        float orow[32];
                        tmem_ld32(t_row, orow);
#pragma unroll
                        for (int i = 0; i < 32; ++i) orow[i] *= al;
                        tmem_st32(t_row, orow);
                        tmem_st_wait();
                    }
                }
                exp_pass();
            }
            // ---- P^T row of this key (16 heads) and the per-head sums of the
            // rounded weights (and of the exact ones for the log-sum-exp)
            uint8_t* prow = sP + (j & 1) * kPBytes + key * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int cc = 2 * hq + c;
                *reinterpret_cast<uint4*>(prow + ((cc ^ (key & 7)) << 4)) =
                    make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            }
#pragma unroll
            for (int i = 0; i < kHPT; i += 2) {
                const float2 r = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i >> 1]));
                acc_r[i] += r.x;
                acc_r[i + 1] += r.y;
            }
            if (LSE && valid) {
#pragma unroll
                for (int i = 0; i < kHPT; ++i) acc_e[i] += ex2(fmaf(sv[i], sl2, -mrow[i]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->p_ready[j & 1]);
        }
        // ---- per-head sums of this warp's 32 keys, then of the four lane quarters
        const float lr_w = warp_transpose_sum16(acc_r, lane);
        if (lane < 16) sLsum[qd * kH + kHPT * hq + lane] = lr_w;
        if (LSE) {
            const float le_w = warp_transpose_sum16(acc_e, lane);
            if (lane < 16) sLsum[4 * kH + qd * kH + kHPT * hq + lane] = le_w;
        }
        if (!ok) *abort = 1;
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(kBN, kH, false, false);
            const uint32_t id_pv = idesc_bf16(kH, kD, true, true);
            const uint64_t qdesc = sw128_desc(smem_u32(sQ), 16, 1024);
            bool ok = true;
            // test hook: a wait that runs out (nothing completes stall_bar)
            if (stall) ok = mbar_wait(&ctl->stall_bar, 0, abort, err, wait_ns);
            auto pv = [&](int jj) -> bool {
                if (!mbar_wait(&ctl->p_ready[jj & 1], (jj >> 1) & 1, abort, err, wait_ns)) return false;
                tc_fence_after();
                const uint64_t pd = sw128_desc(smem_u32(sP + (jj & 1) * kPBytes), kPBytes, 1024);
                const uint64_t vd = sw128_desc(smem_u32(ring + (jj % kStages) * kTileBytes), kHalfK, 1024);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_bf16_ss(t_o, pd + (uint64_t)((kk * 2048) >> 4), vd + (uint64_t)((kk * 2048) >> 4), id_pv,
                                (jj > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&ctl->pv_done);
                mma_commit(&ctl->p_free[jj & 1]);
                mma_commit(&ctl->freeb[jj % kStages]);
                return true;
            };
            for (int j = 0; j < ntile && ok; ++j) {
                if (!mbar_wait(&ctl->full[j % kStages], (j / kStages) & 1, abort, err, wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint64_t kdesc = sw128_desc(smem_u32(ring + (j % kStages) * kTileBytes), 16, 1024);
#pragma unroll
                for (int kq = 0; kq < kD / 16; ++kq) {
                    const uint64_t offk = (uint64_t)(((kq >> 2) * kHalfK + (kq & 3) * 32) >> 4);
                    const uint64_t offq = (uint64_t)(((kq >> 2) * kHalfQ + (kq & 3) * 32) >> 4);
                    mma_bf16_ss(tmem + (j & 1) * 64, kdesc + offk, qdesc + offq, id_qk, kq > 0 ? 1u : 0u);
                }
                mma_commit(&ctl->s_full[j & 1]);
                if (j > 0) ok = pv(j - 1);
            }
            if (ok && ntile > 0 && pv(ntile - 1)) mma_commit(&ctl->o_done);
            // every MMA issued completes before TMEM is released
            mma_commit(&ctl->fin);
            volatile int never = 0;
            mbar_wait(&ctl->fin, 0, &never, err);
        }
        __syncwarp();
    }
    // every copy landed and every MMA completed (the loaders drained their
    // copies, the issuer its MMAs): this warp's part of O into registers
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_arrive();                                // this CTA's ring is free for the peers' pushes
    const bool done = !*abort;
    const bool soft = warp >= kLoadWarps && warp < kMmaWarp;
    float ov[32];                                    // this warp's part of O, kept for the merge
    if (soft) {
        const int qd = warp & 3, hq = (warp - kLoadWarps) >> 2;
        if (done && ntile > 0) tmem_ld32(t_o + ((uint32_t)(32 * qd) << 16) + 32 * hq, ov);
        else {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0.0f;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 256);
    // every CTA of the cluster is past its key ring: the owners' inboxes are free
    cluster_wait();
    // ---- push: partial O rows and states to the CTA that finalises each head
    if (soft) {
        const int qd = warp & 3, hq = (warp - kLoadWarps) >> 2;
        if (lane < 16) {
            const int h = 16 * qd + lane;
            const int own = owner_of(h, C);
            const int hl = h - own * kH / C;
            float* dst = cluster.map_shared_rank(sInO, own) + (size_t)(rank * hmax + hl) * kOS + 32 * hq;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + i) = make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
        }
        const int st = tid - kLoadThreads;
        if (st < kH) {
            float lr = 0.0f, le = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                lr += sLsum[q * kH + st];
                if (LSE) le += sLsum[4 * kH + q * kH + st];
            }
            const int own = owner_of(st, C);
            const int hl = st - own * kH / C;
            cluster.map_shared_rank(sIn, own)[rank * hmax + hl] =
                done ? RowState{sM[st], lr, le} : RowState{-INFINITY, 0.0f, 0.0f};
        }
    }
    cluster_arrive();
    cluster_wait();

    // ---- merge: this CTA finalises heads [rank H / C, (rank + 1) H / C) from its inbox
    const int h_lo = rank * kH / C, h_hi = (rank + 1) * kH / C;
    for (int it = tid; it < (h_hi - h_lo) * (kD / 4); it += kThreads) {
        const int hl = it / (kD / 4), d4 = it - hl * (kD / 4);
        const int hh = h_lo + hl;
        float M = -INFINITY;
        for (int c = 0; c < C; ++c) M = fmaxf(M, sIn[c * hmax + hl].m);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float lr = 0.f, le = 0.f;
        for (int c = 0; c < C; ++c) {
            const RowState s = sIn[c * hmax + hl];
            const float w = s.m == -INFINITY ? 0.0f : exp2f(s.m - M);
            const float4 v = *reinterpret_cast<const float4*>(sInO + (size_t)(c * hmax + hl) * kOS + d4 * 4);
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
            lr = fmaf(w, s.lr, lr);
            le = fmaf(w, s.le, le);
        }
        const float inv = lr > 0.f ? 1.0f / lr : 0.0f;
        T16* out = static_cast<T16*>(a.out) + ((size_t)row * kH + hh) * kD + d4 * 4;
        __nv_bfloat162 w0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        __nv_bfloat162 w1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&w0);
        pk.y = *reinterpret_cast<uint32_t*>(&w1);
        *reinterpret_cast<uint2*>(out) = pk;
        if (LSE && d4 == 0)
            a.lse_out[(size_t)row * kH + hh] = le > 0.f ? (M + log2f(le)) / kLog2e : -INFINITY;
    }
}

long max_keys_dec(const AttnArgs& a) {
    const long comp = ((a.dense ? a.N_cap : a.topk) + kBN - 1) / kBN * kBN;
    const long win = a.window > 0 ? std::min<long>(a.window, a.L_raw) : 0;
    return comp + win;
}

// Row codes a CTA stages: its share of the row's tiles (dealt round-robin).
int chunk_cap_dec(const AttnArgs& a, int C) {
    const long NT = (max_keys_dec(a) + kBN - 1) / kBN;
    return (int)std::max<long>((NT + C - 1) / C * kBN, kBN);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_dec() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// 2D bf16 tensor [rows, 128] with a 128-byte-swizzled box of {64, 128}.
bool make_map_dec(CUtensorMap* m, const void* ptr, uint64_t rows) {
    auto fn = encode_fn_dec();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)std::max<uint64_t>(rows, 1)};
    cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kBN};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <bool LSE>
cudaError_t prepare(int C, size_t smem) {
    auto kern = attn_dec_tc_kernel<LSE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && C > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

// Clusters of C CTAs (one CTA per SM) that can be resident at once; 0 when
// the query fails.  Cached per (device, C, shared-memory size), under a lock
// (host threads may launch concurrently).
int active_clusters(int C, size_t smem) {
    struct Entry {
        int dev, C;
        size_t smem;
        int n;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].C == C && cache[i].smem == smem) return cache[i].n;
    int n = 0;
    if (prepare<false>(C, smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)C, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, attn_dec_tc_kernel<false>, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();
    if (used < 64) cache[used++] = Entry{dev, C, smem, n};
    return n;
}

// Cluster size: the largest C <= 16 whose rows x C CTAs are resident in one
// wave and leave each CTA at least one full tile; 0 when not even C = 1 fits.
int choose_cluster_dec(const AttnArgs& a) {
    const long rows = (long)a.B * a.n_q;
    const long NT = (max_keys_dec(a) + kBN - 1) / kBN;
    for (int C = 16; C >= 1; --C) {
        if (C > 1 && NT < C) continue;
        const int mc = chunk_cap_dec(a, C);
        if (mc > kMaxChunk) return 0;
        if ((long)active_clusters(C, dec_smem(mc).bytes) >= rows) return C;
    }
    return 0;
}

}  // namespace

bool attention_dec_tc_supported(const AttnArgs& a) {
    if (a.dt != DT_BF16 || a.H != kH || a.D != kD || a.vl) return false;
    if (a.B * (long)a.n_q > 65535) return false;
    return choose_cluster_dec(a) > 0;
}

cudaError_t launch_attention_dec_tc(const AttnArgs& a, uint32_t* err, cudaStream_t s) {
    const int C = choose_cluster_dec(a);
    if (C <= 0) return cudaErrorNotSupported;
    const int max_chunk = chunk_cap_dec(a, C);
    const DecSmem L = dec_smem(max_chunk);
    const bool lse = a.lse_out != nullptr;
    // tensor maps of the two caches (any valid address when a cache is empty;
    // not read when the caches are paged)
    CUtensorMap tm_c, tm_w;
    const void* pc = a.kv_c ? a.kv_c : a.kv_raw;
    const void* pw = a.kv_raw ? a.kv_raw : a.kv_c;
    const uint64_t rows_c = a.kv_c ? (uint64_t)a.B * (uint64_t)std::max(a.N_cap, 0) : 1;
    const uint64_t rows_w = a.kv_raw ? (uint64_t)a.B * (uint64_t)std::max(a.L_raw, 0) : 1;
    if (!pc || !pw || !make_map_dec(&tm_c, pc, rows_c) || !make_map_dec(&tm_w, pw, rows_w))
        return cudaErrorInvalidValue;
    cudaError_t e = lse ? prepare<true>(C, L.bytes) : prepare<false>(C, L.bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)(a.B * a.n_q), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L.bytes;
    cfg.stream = s;
    // Programmatic stream serialisation: when the kernel before this one
    // (the decode indexer) signals early, this grid launches and runs its
    // prologue -- TMEM, barriers, Q and the first window tiles -- while that
    // kernel finishes; griddepcontrol.wait orders the read of idx after it.
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const uint64_t wait_ns = wait_limit_ns();
    const int stall = take_stall();
    e = lse ? cudaLaunchKernelEx(&cfg, attn_dec_tc_kernel<true>, tm_c, tm_w, a, max_chunk, err, wait_ns, stall)
            : cudaLaunchKernelEx(&cfg, attn_dec_tc_kernel<false>, tm_c, tm_w, a, max_chunk, err, wait_ns, stall);
    count_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa
