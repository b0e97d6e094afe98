// indexer_split.cu -- stage 2 for few query rows (decode): indexer scores and
// the exact causal top-k, with one row's visible entries split over the CTAs
// of a thread-block cluster.
//
// score[t, s] = sum_h w[t, h] ReLU(qI[t, h] . kI[s]),  s < V(t) = min(floor((t+1)/m), n_entries)
//               (w: gate weights of any sign, 1 when none are given)
// idx[t, :]   = the topk largest scores, equal scores lowest index first, -1 padded
// ("百万上下文从「奢侈品」变「日用品」…" §3.2 indexer score and top-k, §8.2
//  selection without materialising the score matrix; "DS-V4 分析&学习" §1.2,
//  §4 fp8 indexer keys with per-row scales.)
//
// A decode row scores up to N_cap fp8 keys (about 68 bytes each with the
// scale) and keeps only topk, so the step streams the key cache once.  Row r
// is served by a C-CTA cluster; CTA c owns the contiguous entry range
// [c ch, (c+1) ch) and
//   * scores it with e4m3 mma.sync (m16n8k32, fp32 accumulate): the key rows
//     are the A operand loaded straight from global memory, 16 bytes per
//     thread and row, and the query codes of up to 8 heads are the B
//     operand; both sides use the same permutation of the d_I axis, which a
//     dot product does not see.  Each score is kept in shared memory as the
//     bit pattern of a non-negative fp32 value, which orders like the value;
//   * runs a four-digit MSB-first radix select (8-bit digits of the 31-bit
//     non-negative keys) together with its peers: each CTA histograms
//     its own keys, the histograms are summed over DSMEM after a cluster
//     barrier, and every CTA derives the same digit, so all agree on the
//     exact k-th largest key K and on how many keys equal to K are taken;
//   * writes its keys > K and its share of the lowest-index keys == K at
//     offsets given by the counts of the lower-ranked CTAs (ties therefore
//     resolve to the lowest indices across the whole row, and the output is
//     identical from call to call).
// The query row is quantised per head in fp32 exactly as the oracle does
// (scale = amax / 448, codes rounded to nearest even, saturating), after a
// fixed-order Walsh-Hadamard rotation when the keys are of the rotated fp8
// type, unless codes and scales are given.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxHeads = 8;       // one n8 block of the MMA
constexpr int kGroup = 32;         // entries per warp step (two m16 tiles)
constexpr int kMaxChunk = 48 * 1024;   // scores per CTA held in shared memory
static_assert(kWarps == kMaxHeads, "one warp quantises one query head");
// Radix digits of the 32-bit keys (score_key: signed scores with gate
// weights): bits 31-24, 23-16, 15-8 and 7-0.  Four 256-bin rounds measured
// faster than three rounds of 2048 / 1024 bins.
constexpr int kRounds = 4;
__device__ __forceinline__ int round_shift(int rd) { return 24 - 8 * rd; }
__device__ __forceinline__ int round_bits(int) { return 8; }

struct SplitShared {
    unsigned warp_tot[2][kWarps];
    alignas(8) unsigned cnt[2];    // this CTA's keys > K and == K (read by the peers)
    unsigned digit, rank, off_gt, off_eq;
    float qs[kMaxHeads];
    alignas(16) uint8_t qc[kMaxHeads * 128];   // query codes [head][d_I]
};

// D(16x8, f32) += A(16x32, e4m3, row) * B(32x8, e4m3, col)
__device__ __forceinline__ void mma_e4m3(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Sum over the four lanes of a quad (lanes 4g .. 4g+3).
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

template <int NU>
struct Rows {              // one warp step: rows g, g+8, g+16, g+24 of a 32-entry group
    uint4 u[4][NU];
    float sc;              // scale of the entry this thread finalises
};

// Where this CTA's key rows live.  Plain layout: row b * N_cap + e.  Paged:
// the page of entry e comes from the block-table slice staged in shared
// memory (spg, pages p_lo ..), else straight from the block table.
struct RowSrc {
    const uint8_t* kb;     // plain: this element's first key row; paged: the pool
    const float* ksc;      // plain: this element's first scale; paged: the scale pool
    const int* spg;        // paged: staged page ids (or nullptr)
    const int* btrow;      // paged: this element's block-table row
    int p_lo, shift, num_pages;
};

template <bool PAGED>
__device__ __forceinline__ long key_row(const RowSrc& rs, int e) {
    if constexpr (!PAGED) {
        return e;
    } else {
        const int j = e >> rs.shift;
        const int pg = rs.spg ? rs.spg[j - rs.p_lo] : __ldg(rs.btrow + j);
        if (pg < 0 || pg >= rs.num_pages) return -1;
        return ((long)pg << rs.shift) + (e & ((1 << rs.shift) - 1));
    }
}

template <int NU, bool PAGED>
__device__ __forceinline__ void load_rows(Rows<NU>& r, const RowSrc& rs, int base, int hi, int g,
                                          int tq, int wsel) {
    // base is a multiple of 32: with pages of >= 32 entries the whole group
    // lies in one page and one lookup serves it
    const bool one_page = PAGED && rs.shift >= 5;
    const long rbase = one_page ? key_row<PAGED>(rs, base) : 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = base + g + 8 * q;
        const long row = e >= hi ? -1 : (one_page ? (rbase < 0 ? -1 : rbase + (e - base)) : key_row<PAGED>(rs, e));
#pragma unroll
        for (int nu = 0; nu < NU; ++nu)
            r.u[q][nu] = row >= 0 ? __ldcs(reinterpret_cast<const uint4*>(rs.kb + (size_t)row * (64 * NU) + 64 * nu + 16 * tq))
                                  : make_uint4(0u, 0u, 0u, 0u);
    }
    const int ew = base + wsel;
    const long rw = ew >= hi ? -1 : (one_page ? (rbase < 0 ? -1 : rbase + wsel) : key_row<PAGED>(rs, ew));
    r.sc = rw >= 0 ? __ldcs(rs.ksc + rw) : 0.0f;
}

constexpr int kPageSlots = 1024;   // block-table entries a paged CTA stages in shared memory

// Resident CTAs per SM the register budget is sized for (d_I = 64: four).
template <int NU>
constexpr int min_blocks() { return NU == 1 ? 4 : 2; }

template <int QD, int NU, bool PAGED>
__global__ void __launch_bounds__(kThreads, min_blocks<NU>()) indexer_split_kernel(IndexerArgs a) {
    extern __shared__ __align__(16) unsigned dyn[];   // [2][256] histograms, [ch] keys, (paged) page ids
    unsigned* hist_buf = dyn;
    unsigned* keys = dyn + 2 * 256;                   // score keys of this CTA's entries
    __shared__ SplitShared sh;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    constexpr int d = 64 * NU;

    const int row = blockIdx.y;
    const int b = row / a.n_q;
    const int H = a.H_I, topk = a.topk;
    int* out = a.idx_out + (size_t)row * topk;
    const int t = a.q_pos ? a.q_pos[row] : a.pos0 + (row - b * a.n_q);
    const int ne = clampi(a.n_entries ? a.n_entries[b] : a.N_cap, 0, a.N_cap);
    const int V = t < 0 ? 0 : min((t + 1) / a.m, ne);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (V <= topk) {        // every CTA of the cluster takes this branch together
        for (int j = rank * kThreads + tid; j < topk; j += C * kThreads) out[j] = j < V ? j : -1;
        return;
    }
    const int ch = ((V + C - 1) / C + kGroup - 1) / kGroup * kGroup;
    const int lo = min(V, rank * ch), hi = min(V, lo + ch);
    const int nloc = hi - lo;

    // ---- query codes and per-head scales (heads >= H_I are zero)
    if constexpr (QD == DT_E4M3) {
        const uint8_t* src = static_cast<const uint8_t*>(a.qI) + (size_t)row * H * d;
        for (int p = tid; p < kMaxHeads * d; p += kThreads) sh.qc[p] = p < H * d ? src[p] : 0;
        if (tid < kMaxHeads)
            sh.qs[tid] = tid < H ? a.qI_scale[(size_t)row * H + tid] *
                                       (a.qI_weight ? a.qI_weight[(size_t)row * H + tid] : 1.0f)
                                 : 0.0f;
    } else {
        const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(a.qI) + (size_t)row * H * d;
        const int h = warp;   // kWarps == kMaxHeads
        if (h < H) {
            constexpr int J = d / 32;          // this lane holds elements lane + 32 j
            float v[J];
#pragma unroll
            for (int j = 0; j < J; ++j) v[j] = __bfloat162float(src[h * d + lane + 32 * j]);
            if (a.kI_dt == DT_E4M3H) {
                // Walsh-Hadamard butterflies in stride order: strides 1..16
                // pair lane with lane ^ s (the lower lane holds the left
                // operand), strides 32, 64 pair this lane's own elements.
#pragma unroll
                for (int sl = 1; sl < 32; sl <<= 1) {
                    const bool hi = (lane & sl) != 0;
#pragma unroll
                    for (int j = 0; j < J; ++j) {
                        const float pv = __shfl_xor_sync(0xffffffffu, v[j], sl);
                        v[j] = hi ? pv - v[j] : v[j] + pv;
                    }
                }
#pragma unroll
                for (int sj = 1; sj < J; sj <<= 1) {
#pragma unroll
                    for (int j = 0; j < J; ++j) {
                        if (j & sj) continue;
                        const float x0 = v[j], x1 = v[j + sj];
                        v[j] = x0 + x1;
                        v[j + sj] = x0 - x1;
                    }
                }
#pragma unroll
                for (int j = 0; j < J; ++j) v[j] = v[j] * a.hnorm;
            }
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < J; ++j) amax = fmaxf(amax, fabsf(v[j]));
            for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
#pragma unroll
            for (int j = 0; j < J; ++j) sh.qc[h * d + lane + 32 * j] = e4m3_code(__fdiv_rn(v[j], scale));
            if (lane == 0) sh.qs[h] = a.qI_weight ? scale * a.qI_weight[(size_t)row * H + h] : scale;
        } else {
            for (int c = lane; c < d; c += 32) sh.qc[h * d + c] = 0;
            if (lane == 0) sh.qs[h] = 0.0f;
        }
    }
    // ---- paged caches: this CTA's slice of the block table into shared memory
    bool pages_staged = false;
    const int ch_alloc = max((a.N_cap + C - 1) / C + kGroup - 1, kGroup) / kGroup * kGroup;
    if constexpr (PAGED) {
        const int p_lo = lo >> a.pages.page_shift;
        const int np = hi > lo ? ((hi - 1) >> a.pages.page_shift) - p_lo + 1 : 0;
        pages_staged = np <= kPageSlots;
        if (pages_staged) {
            int* spg = reinterpret_cast<int*>(keys + ch_alloc);
            const int* btrow = a.pages.bt + (size_t)b * a.pages.max_pages;
            for (int i = tid; i < np; i += kThreads) spg[i] = btrow[p_lo + i];
        }
    }
    __syncthreads();

    // ---- scores of [lo, hi)
    {
        const int g = lane >> 2, tq = lane & 3;
        // B fragments: head g, the 16 query bytes at [64 nu + 16 tq, +16)
        uint32_t bq[NU][4];
#pragma unroll
        for (int nu = 0; nu < NU; ++nu) {
            const uint4 v = *reinterpret_cast<const uint4*>(sh.qc + g * d + 64 * nu + 16 * tq);
            bq[nu][0] = v.x; bq[nu][1] = v.y; bq[nu][2] = v.z; bq[nu][3] = v.w;
        }
        const float qs0 = sh.qs[2 * tq], qs1 = sh.qs[2 * tq + 1];
        RowSrc src;
        src.kb = static_cast<const uint8_t*>(a.kI);
        src.ksc = a.kI_scale;
        if constexpr (!PAGED) {
            src.kb += (size_t)b * a.N_cap * d;
            src.ksc += (size_t)b * a.N_cap;
        } else {
            src.btrow = a.pages.bt + (size_t)b * a.pages.max_pages;
            src.shift = a.pages.page_shift;
            src.num_pages = a.pages.num_pages;
            src.p_lo = lo >> src.shift;
            src.spg = pages_staged ? reinterpret_cast<const int*>(keys + ch_alloc) : nullptr;
        }
        const int wsel = (tq >> 1) * 16 + (tq & 1) * 8 + g;   // the entry this thread finalises
        const int step = kWarps * kGroup;
        Rows<NU> cur, nxt;
        int base = lo + warp * kGroup;
        if (base < hi) load_rows<NU, PAGED>(cur, src, base, hi, g, tq, wsel);
        for (; base < hi; base += step) {
            if (base + step < hi) load_rows<NU, PAGED>(nxt, src, base + step, hi, g, tq, wsel);
            float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int nu = 0; nu < NU; ++nu) {
                // A rows g / g+8 (tile 0) and g+16 / g+24 (tile 1); k slots 4tq.. <- bytes 16tq..
                mma_e4m3(c0, cur.u[0][nu].x, cur.u[1][nu].x, cur.u[0][nu].y, cur.u[1][nu].y, bq[nu][0], bq[nu][1]);
                mma_e4m3(c0, cur.u[0][nu].z, cur.u[1][nu].z, cur.u[0][nu].w, cur.u[1][nu].w, bq[nu][2], bq[nu][3]);
                mma_e4m3(c1, cur.u[2][nu].x, cur.u[3][nu].x, cur.u[2][nu].y, cur.u[3][nu].y, bq[nu][0], bq[nu][1]);
                mma_e4m3(c1, cur.u[2][nu].z, cur.u[3][nu].z, cur.u[2][nu].w, cur.u[3][nu].w, bq[nu][2], bq[nu][3]);
            }
            // heads 2tq, 2tq+1 of entries g, g+8, g+16, g+24
            const float p0 = quad_sum(fmaf(qs0, relu0(c0[0]), qs1 * relu0(c0[1])));
            const float p1 = quad_sum(fmaf(qs0, relu0(c0[2]), qs1 * relu0(c0[3])));
            const float p2 = quad_sum(fmaf(qs0, relu0(c1[0]), qs1 * relu0(c1[1])));
            const float p3 = quad_sum(fmaf(qs0, relu0(c1[2]), qs1 * relu0(c1[3])));
            const float mine = tq == 0 ? p0 : (tq == 1 ? p1 : (tq == 2 ? p2 : p3));
            const int e = base + wsel;
            if (e < hi) keys[e - lo] = score_key(mine * cur.sc);
            cur = nxt;
        }
    }
    __syncthreads();

    // ---- cluster-wide radix select: exact k-th largest key K, and how many == K to take.
    // Keys are score_key() images of the fp32 scores; four 8-bit digits
    // settle all 32 bits.
    unsigned prefix = 0, pmask = 0, need = (unsigned)topk;
#pragma unroll 1
    for (int rd = 0; rd < kRounds; ++rd) {
        const int shift = round_shift(rd);
        const int nbins = 1 << round_bits(rd);
        const unsigned dmask = (unsigned)nbins - 1u;
        unsigned* hist = hist_buf + (rd & 1) * 256;    // the other buffer may still be read by peers
        for (int i = tid; i < nbins; i += kThreads) hist[i] = 0;
        __syncthreads();
        // warp-aggregated: lanes with the same digit add once (the leading
        // digits of similar scores collide heavily)
        for (int i0 = 0; i0 < nloc; i0 += kThreads) {
            const int i = i0 + tid;
            const unsigned k = i < nloc ? keys[i] : 0u;
            const bool take = i < nloc && (k & pmask) == prefix;
            const unsigned d = take ? (k >> shift) & dmask : 0xffffffffu;
            const unsigned peers = __match_any_sync(0xffffffffu, d);
            if (take && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (unsigned)__popc(peers));
        }
        cluster.sync();
        // thread t owns the bpt bins just below nbins - bpt t (highest digits first)
        const int bpt = nbins / kThreads;            // 1, 4 or 8
        const int b0 = nbins - bpt * (tid + 1);
        unsigned cnt[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) cnt[i] = 0;
#pragma unroll
        for (int c = 0; c < 16; ++c) {               // every peer's bins requested before use
            if (c < C) {
                const unsigned* ph = cluster.map_shared_rank(hist, c) + b0;
                if (bpt == 1) {
                    cnt[0] += *ph;
                } else {
                    const uint4 lo4 = *reinterpret_cast<const uint4*>(ph);
                    cnt[0] += lo4.x; cnt[1] += lo4.y; cnt[2] += lo4.z; cnt[3] += lo4.w;
                    if (bpt == 8) {
                        const uint4 hi4 = *reinterpret_cast<const uint4*>(ph + 4);
                        cnt[4] += hi4.x; cnt[5] += hi4.y; cnt[6] += hi4.z; cnt[7] += hi4.w;
                    }
                }
            }
        }
        unsigned sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += cnt[i];
        // block-wide inclusive scan of the per-thread sums, in thread order
        unsigned incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) sh.warp_tot[0][warp] = incl;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            if (w < warp) incl += sh.warp_tot[0][w];
        const unsigned excl = incl - sum;
        if (excl < need && need <= incl) {
            unsigned run = excl;
            // this thread's bins in descending digit order: b0 + bpt - 1 down to b0
#pragma unroll
            for (int i = 7; i >= 0; --i) {
                if (i < bpt && run < need && need <= run + cnt[i]) {
                    sh.digit = (unsigned)(b0 + i);
                    sh.rank = need - run;
                }
                if (i < bpt) run += cnt[i];
            }
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        pmask |= dmask << shift;
        need = sh.rank;
        __syncthreads();     // warp_tot and digit are rewritten next round
    }
    const unsigned K = prefix;
    const unsigned need_eq = need;                 // >= 1 keys equal to K are taken
    const unsigned n_gt = (unsigned)topk - need_eq;

    // ---- each warp owns a contiguous block of this CTA's keys; count, then emit in order
    const int per = ((nloc + kWarps - 1) / kWarps + 31) & ~31;
    const int w_lo = min(nloc, warp * per), w_hi = min(nloc, w_lo + per);
    {
        unsigned gt = 0, eq = 0;
        for (int i = w_lo + lane; i < w_hi; i += 32) {
            const unsigned k = keys[i];
            gt += k > K;
            eq += k == K;
        }
        for (int off = 16; off; off >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, off);
            eq += __shfl_xor_sync(0xffffffffu, eq, off);
        }
        if (lane == 0) { sh.warp_tot[0][warp] = gt; sh.warp_tot[1][warp] = eq; }
        __syncthreads();
        if (tid == 0) {
            unsigned sg = 0, se = 0;
            for (int w = 0; w < kWarps; ++w) { sg += sh.warp_tot[0][w]; se += sh.warp_tot[1][w]; }
            sh.cnt[0] = sg;
            sh.cnt[1] = se;
        }
        cluster.sync();
        if (warp == 0) {     // lane c reads the counts of peer c < rank
            uint2 pc = make_uint2(0u, 0u);
            if (lane < rank) pc = *reinterpret_cast<const uint2*>(cluster.map_shared_rank(sh.cnt, lane));
            for (int off = 16; off; off >>= 1) {
                pc.x += __shfl_xor_sync(0xffffffffu, pc.x, off);
                pc.y += __shfl_xor_sync(0xffffffffu, pc.y, off);
            }
            if (lane == 0) { sh.off_gt = pc.x; sh.off_eq = pc.y; }
        }
        __syncthreads();
    }

    // ---- ordered emission: keys > K at [0, n_gt), the first need_eq keys == K after them
    unsigned run_gt = sh.off_gt, run_eq = sh.off_eq;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
        if (w < warp) { run_gt += sh.warp_tot[0][w]; run_eq += sh.warp_tot[1][w]; }
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = w_lo; base < w_hi; base += 32) {
        const int i = base + lane;
        const unsigned k = i < w_hi ? keys[i] : 0u;
        const bool gt = i < w_hi && k > K;
        const bool eq = i < w_hi && k == K;
        const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
        if (gt) {
            const unsigned r = run_gt + __popc(bg & lt_mask);
            if (r < n_gt) out[r] = lo + i;
        }
        if (eq) {
            const unsigned r = run_eq + __popc(be & lt_mask);
            if (r < need_eq) out[n_gt + r] = lo + i;
        }
        run_gt += __popc(bg);
        run_eq += __popc(be);
    }
    cluster.sync();     // keep this CTA's shared memory alive until every peer has read it
    // This CTA's indices are written: a kernel launched after this one with
    // programmatic serialisation (the decode attention) may begin its
    // prologue; it still waits for this grid's completion before reading idx.
    // Signalled last, so every CTA of this grid already holds its SM.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// Cluster size: the largest power of two <= 16 with rows x C CTAs within one
// wave of resident CTAs and at least 256 entries per CTA; larger if a row's
// share would not fit shared memory.
int choose_cluster(const IndexerArgs& a) {
    const long rows = (long)a.B * a.n_q;
    const long slots = (long)num_sms() * (a.d_I == 64 ? min_blocks<1>() : min_blocks<2>());
    int C = 1;
    while (2 * C <= 16 && rows * 2 * C <= slots && a.N_cap / (2 * C) >= 256) C *= 2;
    while (C < 16 && ((long)a.N_cap + C - 1) / C > kMaxChunk) C *= 2;
    return C;
}

long chunk_cap(const IndexerArgs& a, int C) {
    return std::max<long>(((long)a.N_cap + C - 1) / C + kGroup - 1, kGroup) / kGroup * kGroup;
}

template <int QD, int NU, bool PAGED>
cudaError_t launch_t(const IndexerArgs& a, cudaStream_t s) {
    const int C = choose_cluster(a);
    const size_t smem = sizeof(unsigned) * ((size_t)chunk_cap(a, C) + 2 * 256 + (PAGED ? kPageSlots : 0));
    auto kern = indexer_split_kernel<QD, NU, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (C > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)(a.B * a.n_q), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    count_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

bool indexer_split_supported(const IndexerArgs& a) {
    if ((a.kI_dt != DT_E4M3 && a.kI_dt != DT_E4M3H) || a.kI_scale == nullptr) return false;
    if (!(a.qI_dt == DT_BF16 || (a.qI_dt == DT_E4M3 && a.qI_scale != nullptr))) return false;
    if ((a.d_I != 64 && a.d_I != 128) || a.H_I < 1 || a.H_I > kMaxHeads) return false;
    if ((long)a.B * a.n_q > 65535) return false;
    return chunk_cap(a, choose_cluster(a)) <= kMaxChunk;
}

template <bool PAGED>
cudaError_t launch_paging(const IndexerArgs& a, cudaStream_t s) {
    if (a.qI_dt == DT_E4M3)
        return a.d_I == 64 ? launch_t<DT_E4M3, 1, PAGED>(a, s) : launch_t<DT_E4M3, 2, PAGED>(a, s);
    return a.d_I == 64 ? launch_t<DT_BF16, 1, PAGED>(a, s) : launch_t<DT_BF16, 2, PAGED>(a, s);
}

cudaError_t launch_indexer_split(const IndexerArgs& a, cudaStream_t s) {
    return a.pages.bt ? launch_paging<true>(a, s) : launch_paging<false>(a, s);
}

}  // namespace csa
